/*
 * mx_oracle.c -- plain, slow, single-threaded CPU oracle for the MixLLM
 * mixed-precision quantized linear layer (W4.4A8).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library; both sides are written independently from the method's text.
 *
 * Sources (MixLLM: "LLM Quantization with Global Mixed-precision between
 * Output-features and Highly-efficient System Design", paper digest page):
 *   - affine quantizer  X_q = clamp(round(X/s) + z, range), X' = (X_q - z) s
 *       (section 2.1, "quantization principle")
 *   - symmetric quantizer X_q = clamp(round(W/s), range), X' = X_q s
 *       (section 2.1, "quantization scheme")
 *   - 8-bit symmetric activations, 8-bit symmetric / 4-bit asymmetric
 *     group-wise weights, group 128 (section 3.1.2; section 4 setup)
 *   - output-feature mixed precision: every output row is an independent
 *     sub-problem, results gathered into one Y (section 3.1.1, Figure 1)
 *   - two-step dequantization: (W_q - z) times A_q on integers per group,
 *     then both scales per group (section 3.3); W_q, z are uint4, s_w, s_a
 *     are float16 (section 3.3)
 *   - restricted symmetric range +-(2^(b-1) - 1) (SBVR page, section 2.1)
 *
 * Readings where the text is silent:
 *   - symmetric range [-127, 127], s = absmax / 127
 *   - the 4-bit range [lo, hi] always contains 0, so z fits uint4
 *   - round() is round-half-to-even
 *   - scales are computed in fp32, rounded to fp16 (nearest-even) and the
 *      ROUNDED fp16 value is the one used to quantize
 *   - a zero (or fp16-underflowed) scale becomes 1.0; an fp16 overflow
 *      saturates to 65504
 *   - fp32 quantization decisions: amax/127, (hi-lo)/15, x/s, -lo/s are
 *      each one IEEE fp32 operation; everything after the integer codes is
 *      exact integer (int64) or fp64 arithmetic here
 *
 * Parity of every function below is pinned by CPU tests against closed
 * forms, brute force, textbook special cases and library conversions.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (x86-64 evaluates float in SSE single precision, FLT_EVAL_METHOD == 0).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(__FLT_EVAL_METHOD__) && __FLT_EVAL_METHOD__ != 0
#error "the oracle needs IEEE single-precision evaluation of float expressions"
#endif

/* ------------------------------------------------------------------------ */
/* IEEE-754 binary16 rounding, written from the format's definition:        */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; normal numbers  */
/* have exponents -14..15, subnormals a fixed quantum of 2^-24; the largest */
/* finite value is 65504; round-to-nearest, ties-to-even.                   */
/* ------------------------------------------------------------------------ */

/* nearest binary16 value of v, as a double (exact); overflow gives +-inf */
double mxo_fp16_round(double v)
{
    if (v != v) return v;
    double a = fabs(v);
    if (a == 0.0) return v;
    int e;
    frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
    int E = e - 1;                /* unbiased exponent of a */
    if (E < -14) E = -14;         /* subnormal binade: quantum stays 2^-24 */
    double quantum = ldexp(1.0, E - 10);
    double r = rint(a / quantum) * quantum;   /* a/quantum is exact */
    if (r >= 65536.0) r = INFINITY;           /* beyond 65504 + half ulp */
    return copysign(r, v);
}

/* bit pattern of a value that is already exactly representable in binary16 */
uint16_t mxo_fp16_bits_of(double r)
{
    uint16_t sign = signbit(r) ? 0x8000u : 0u;
    double a = fabs(r);
    if (a != a) return 0x7E00u;
    if (isinf(a)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {                       /* subnormal */
        return (uint16_t)(sign | (uint16_t)(a / ldexp(1.0, -24)));
    }
    int e;
    double f = frexp(a, &e);                         /* a = f 2^e, f in [0.5,1) */
    int E = e - 1;
    uint16_t frac = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | frac);
}

/* value of a binary16 bit pattern */
double mxo_fp16_value(uint16_t h)
{
    int s = (h >> 15) & 1, E = (h >> 10) & 31, f = h & 1023;
    double v;
    if (E == 31) v = f ? NAN : INFINITY;
    else if (E == 0) v = ldexp((double)f, -24);
    else v = ldexp(1024.0 + f, E - 25);
    return s ? -v : v;
}

/* The fp16 scale the quantizers use: the fp32 scale rounded to fp16,      */
/* saturated at 65504; zero (or an fp16 underflow) becomes 1.  The paper   */
/* fixes only the fp16 type of the scales (MixLLM section 3.3).           */
static float scale_to_fp16(float s32, uint16_t *bits)
{
    double s16 = mxo_fp16_round((double)s32);
    if (s16 > 65504.0) s16 = 65504.0;          /* fp16 overflow saturates */
    if (s16 == 0.0) s16 = 1.0;                 /* degenerate group */
    *bits = mxo_fp16_bits_of(s16);
    return (float)s16;                         /* exact */
}

static float clampf_(float v, float lo, float hi)
{
    return v < lo ? lo : (v > hi ? hi : v);
}

/* ------------------------------------------------------------------------ */
/* Symmetric 8-bit quantizer (section 2.1 "quantization scheme", range      */
/* +-127; the range is left open there): s = fp16(absmax/127),            */
/* q = clamp(round(x/s), -127, 127).                                        */
/* ------------------------------------------------------------------------ */
void mxo_quant_sym8(const float *x, int n, int8_t *q, uint16_t *s_bits)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s = scale_to_fp16(amax / 127.0f, s_bits);
    for (int i = 0; i < n; ++i) {
        float r = rintf(x[i] / s);
        q[i] = (int8_t)clampf_(r, -127.0f, 127.0f);
    }
}

/* ------------------------------------------------------------------------ */
/* Asymmetric 4-bit quantizer (section 2.1 affine form; z is uint4 per      */
/* section 3.3, so the range includes 0):                                   */
/*   lo = min(0, min x), hi = max(0, max x), s = fp16((hi - lo)/15),         */
/*   z = clamp(round(-lo/s), 0, 15), q = clamp(round(x/s) + z, 0, 15).       */
/* ------------------------------------------------------------------------ */
void mxo_quant_asym4(const float *x, int n, uint8_t *q, uint8_t *z, uint16_t *s_bits)
{
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < n; ++i) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    float range = hi - lo;
    float s = scale_to_fp16(range / 15.0f, s_bits);
    float zf = clampf_(rintf(-lo / s), 0.0f, 15.0f);
    *z = (uint8_t)zf;
    for (int i = 0; i < n; ++i) {
        float r = rintf(x[i] / s) + zf;
        q[i] = (uint8_t)clampf_(r, 0.0f, 15.0f);
    }
}

/* ------------------------------------------------------------------------ */
/* Activation quantization: 8-bit symmetric per token (act_group == 0) or   */
/* per group of act_group columns (section 3.1.2 names group-wise scales;  */
/* the measured configuration uses one scale per token).                    */
/* X: [M][ldx] fp32.  Aq: [M][K] int8.  s_a: [M] (per token) or [M][K/ag].  */
/* Returns 0, or -1 on bad arguments.                                       */
/* ------------------------------------------------------------------------ */
int mxo_quant_act(const float *X, int M, int K, int ldx, int act_group,
                  int8_t *Aq, uint16_t *s_a)
{
    if (M < 0 || K <= 0 || ldx < K) return -1;
    int ag = act_group == 0 ? K : act_group;
    if (ag <= 0 || K % ag) return -1;
    int na = K / ag;
    for (int m = 0; m < M; ++m)
        for (int j = 0; j < na; ++j)
            mxo_quant_sym8(X + (size_t)m * ldx + (size_t)j * ag, ag,
                           Aq + (size_t)m * K + (size_t)j * ag, s_a + (size_t)m * na + j);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Packing into the CANONICAL form (the compare target of the GPU blob):    */
/*   perm[N]           packed row j -> original row; the 8-bit rows first   */
/*                     in ascending original index, then the 4-bit rows in  */
/*                     ascending original index (section 3.1.1, Figure 1:   */
/*                     independent sub-problems, gathered afterwards)       */
/*   codes8[N8][K]     int8, scales8[N8][G] fp16 bits                        */
/*   codes4[N4][K]     uint8 (one code per byte), zeros4[N4][G] uint8,      */
/*                     scales4[N4][G] fp16 bits                              */
/* W: [N][ldw] fp32; is8[N]: nonzero = salient row kept at 8 bits.          */
/* Returns N8 (>= 0), or -1 on bad arguments.                               */
/* ------------------------------------------------------------------------ */
int mxo_pack(const float *W, int N, int K, int ldw, int group, const uint8_t *is8,
             int32_t *perm, int8_t *codes8, uint16_t *scales8,
             uint8_t *codes4, uint8_t *zeros4, uint16_t *scales4)
{
    if (N < 0 || K <= 0 || ldw < K || group <= 0 || K % group) return -1;
    int G = K / group;
    int n8 = 0;
    for (int n = 0; n < N; ++n) if (is8[n]) perm[n8++] = n;
    int j = n8;
    for (int n = 0; n < N; ++n) if (!is8[n]) perm[j++] = n;
    for (int r = 0; r < n8; ++r) {
        const float *w = W + (size_t)perm[r] * ldw;
        for (int g = 0; g < G; ++g)
            mxo_quant_sym8(w + (size_t)g * group, group,
                           codes8 + (size_t)r * K + (size_t)g * group,
                           scales8 + (size_t)r * G + g);
    }
    for (int r = 0; r < N - n8; ++r) {
        const float *w = W + (size_t)perm[n8 + r] * ldw;
        for (int g = 0; g < G; ++g)
            mxo_quant_asym4(w + (size_t)g * group, group,
                            codes4 + (size_t)r * K + (size_t)g * group,
                            zeros4 + (size_t)r * G + g,
                            scales4 + (size_t)r * G + g);
    }
    return n8;
}

/* packed index of every original row (inverse of perm) */
static int32_t *invert_perm(const int32_t *perm, int N)
{
    int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!inv) return NULL;
    for (int j = 0; j < N; ++j) inv[perm[j]] = j;
    return inv;
}

/* integer weight (W_q - z) of packed row j at column k: the first step of  */
/* the two-step dequantization (section 3.3); z = 0 for the 8-bit rows       */
static int wint(int j, int k, int K, int group, int n8, const int8_t *codes8,
                const uint8_t *codes4, const uint8_t *zeros4)
{
    if (j < n8) return (int)codes8[(size_t)j * K + k];
    int r = j - n8, G = K / group;
    return (int)codes4[(size_t)r * K + k] - (int)zeros4[(size_t)r * G + k / group];
}

static double wscale(int j, int g, int G, int n8, const uint16_t *scales8,
                     const uint16_t *scales4)
{
    if (j < n8) return mxo_fp16_value(scales8[(size_t)j * G + g]);
    return mxo_fp16_value(scales4[(size_t)(j - n8) * G + g]);
}

/* ------------------------------------------------------------------------ */
/* Per-group integer partials (section 3.3 step one):                        */
/*   P[m][n][g] = sum_{k in group g} Aq[m][k] * (W_q[n][k] - z[n][g])        */
/* in int64, n in ORIGINAL row order.  Returns the largest |P| seen, or -1.  */
/* ------------------------------------------------------------------------ */
int64_t mxo_partials(const int8_t *Aq, int M, int K, int group, int N,
                     const int32_t *perm, int n8,
                     const int8_t *codes8, const uint8_t *codes4, const uint8_t *zeros4,
                     int64_t *P)
{
    if (M < 0 || K <= 0 || group <= 0 || K % group || N < 0) return -1;
    int G = K / group;
    int32_t *inv = invert_perm(perm, N);
    if (!inv) return -1;
    int64_t pmax = 0;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            int j = inv[n];
            for (int g = 0; g < G; ++g) {
                int64_t acc = 0;
                for (int k = g * group; k < (g + 1) * group; ++k)
                    acc += (int64_t)Aq[(size_t)m * K + k] *
                           (int64_t)wint(j, k, K, group, n8, codes8, codes4, zeros4);
                P[((size_t)m * N + n) * G + g] = acc;
                if (llabs(acc) > pmax) pmax = llabs(acc);
            }
        }
    free(inv);
    return pmax;
}

/* ------------------------------------------------------------------------ */
/* Y = dequant(Xq) . dequant(Wq)^T, fp64, at the listed (m, n) pairs        */
/* (n in original row order), two ways that must agree:                     */
/*  Y_def: the plain definition, sum_k (Aq s_a)[m][k] * ((W_q - z) s_w)[n][k]*/
/*         (section 2.1 dequantization applied to both operands)            */
/*  Y_two: the two-step form of section 3.3,                                */
/*         sum_g s_a[m][g] s_w[n][g] P[m][n][g]  (s_a per token when        */
/*         act_group == 0)                                                  */
/* pairs == NULL means every (m, n), written row-major [M][N].              */
/* Returns 0, or -1 on bad arguments.                                       */
/* ------------------------------------------------------------------------ */
int mxo_gemm(const int8_t *Aq, const uint16_t *s_a, int act_group, int M, int K,
             int group, int N, const int32_t *perm, int n8,
             const int8_t *codes8, const uint16_t *scales8,
             const uint8_t *codes4, const uint8_t *zeros4, const uint16_t *scales4,
             const int32_t *pair_m, const int32_t *pair_n, long n_pairs,
             double *Y_def, double *Y_two)
{
    if (M < 0 || K <= 0 || group <= 0 || K % group || N < 0) return -1;
    if (act_group != 0 && act_group != group) return -1;
    int G = K / group;
    int na = act_group == 0 ? 1 : G;
    int32_t *inv = invert_perm(perm, N);
    if (!inv) return -1;
    long total = pair_m ? n_pairs : (long)M * N;
    for (long t = 0; t < total; ++t) {
        int m = pair_m ? pair_m[t] : (int)(t / (N > 0 ? N : 1));
        int n = pair_m ? pair_n[t] : (int)(t % (N > 0 ? N : 1));
        if (m < 0 || m >= M || n < 0 || n >= N) { free(inv); return -1; }
        int j = inv[n];
        double ydef = 0.0, ytwo = 0.0;
        for (int g = 0; g < G; ++g) {
            double sa = mxo_fp16_value(s_a[(size_t)m * na + (na == 1 ? 0 : g)]);
            double sw = wscale(j, g, G, n8, scales8, scales4);
            int64_t p = 0;
            for (int k = g * group; k < (g + 1) * group; ++k) {
                int a = Aq[(size_t)m * K + k];
                int w = wint(j, k, K, group, n8, codes8, codes4, zeros4);
                ydef += ((double)a * sa) * ((double)w * sw);
                p += (int64_t)a * (int64_t)w;
            }
            ytwo += sa * sw * (double)p;
        }
        Y_def[t] = ydef;
        Y_two[t] = ytwo;
    }
    free(inv);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Channel saliency of the global precision search (MixLLM section 3.2,     */
/* Eq. 4 with the gradient of one calibration batch, as Algorithm 1 uses    */
/* it): per output row n of one layer,                                     */
/*   dW = dequant(quantize(W)) - W   (quantize: the 4-bit asymmetric group  */
/*        quantizer above, the precision a row falls to when it is not      */
/*        selected; no other quantizer is named for this step),            */
/*   S1 = sum_k G[n,k] * dW[n,k],  S[n] = | S1 + S1^2 / 2 |.                */
/* W, G: [N][ld] fp32.  S: [N] fp64.  All arithmetic after the codes is     */
/* fp64.  Returns 0, or -1 on bad arguments.                                */
/* ------------------------------------------------------------------------ */
int mxo_saliency(const float *W, int ldw, const float *G, int ldg, int N, int K, int group, double *S)
{
    if (N < 0 || K <= 0 || group <= 0 || K % group != 0 || ldw < K || ldg < K) return -1;
    uint8_t *q = (uint8_t *)malloc((size_t)group);
    if (!q) return -1;
    for (int n = 0; n < N; ++n) {
        double s1 = 0.0;
        for (int g0 = 0; g0 < K; g0 += group) {
            const float *w = W + (size_t)n * ldw + g0;
            const float *gr = G + (size_t)n * ldg + g0;
            uint8_t z;
            uint16_t sb;
            mxo_quant_asym4(w, group, q, &z, &sb);
            const double s = mxo_fp16_value(sb);
            for (int k = 0; k < group; ++k) {
                const double dq = ((double)q[k] - (double)z) * s;   /* dequantized weight */
                s1 += (double)gr[k] * (dq - (double)w[k]);
            }
        }
        S[n] = fabs(s1 + 0.5 * s1 * s1);
    }
    free(q);
    return 0;
}

/* ======================================================================== */
/* Block-wise bit widths (ScaleBITS blog page: section 1.2.2, the hardware- */
/* aligned block partition with one bit width per 64 x 128 block; section   */
/* 3.2, the block-wise layout with 2-bit metadata recording each block's    */
/* width; section 4.2, the width search space {1, 2, 3, 4, 6, 8}).          */
/*                                                                          */
/* Readings (the page gives no quantizer and no layout beyond that):        */
/*  - a block is 64 output rows x 128 input columns; the last row block may */
/*    be short; K is a multiple of 128;                                     */
/*  - the 2-bit code of a block indexes a four-entry width table of the     */
/*    layer; the codes are stored four to a byte, block i in bits           */
/*    2(i mod 4) of byte i / 4, blocks in row-major (row block, column      */
/*    block) order;                                                         */
/*  - inside a block each row's 128 weights are one group with its own fp16 */
/*    scale (and zero), as MixLLM's group-wise weights;                     */
/*  - b = 8: the symmetric 8-bit quantizer above (z = 0); b < 8: the        */
/*    asymmetric b-bit form of the 4-bit quantizer above, levels            */
/*    0 .. 2^b - 1.  So q - z always fits int8 and the same two-step int8   */
/*    dequantization applies to every block.                                */
/* ======================================================================== */

/* Asymmetric b-bit quantizer, 1 <= b <= 7 (b = 4 is mxo_quant_asym4):       */
/*   qmax = 2^b - 1, lo = min(0, min x), hi = max(0, max x),                */
/*   s = fp16((hi - lo)/qmax), z = clamp(round(-lo/s), 0, qmax),            */
/*   q = clamp(round(x/s) + z, 0, qmax).                                    */
int mxo_quant_asym(const float *x, int n, int bits, uint8_t *q, uint8_t *z, uint16_t *s_bits)
{
    if (n <= 0 || bits < 1 || bits > 7) return -1;
    const float qmax = (float)((1 << bits) - 1);
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < n; ++i) {
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    float range = hi - lo;
    float s = scale_to_fp16(range / qmax, s_bits);
    float zf = clampf_(rintf(-lo / s), 0.0f, qmax);
    *z = (uint8_t)zf;
    for (int i = 0; i < n; ++i) {
        float r = rintf(x[i] / s) + zf;
        q[i] = (uint8_t)clampf_(r, 0.0f, qmax);
    }
    return 0;
}

#define MXO_BLK_ROWS 64
#define MXO_BLK_COLS 128

/* the width of block (rb, kb) from the packed 2-bit codes and the table */
static int block_bits(const uint8_t *meta, const uint8_t *table, int KB, int rb, int kb)
{
    long i = (long)rb * KB + kb;
    return table[(meta[i >> 2] >> (2 * (i & 3))) & 3];
}

/* Quantize W [N][ldw] fp32 block by block.  table: four widths, each in    */
/* 1..8.  meta: ceil(NB * KB / 4) bytes of 2-bit codes, NB = ceil(N / 64),  */
/* KB = K / 128.  Out, in original row order: q [N][K] int16 (the code:     */
/* -127..127 for 8-bit blocks, 0..2^b - 1 otherwise), zeros [N][KB] uint8   */
/* (0 for 8-bit blocks), scales [N][KB] fp16 bits.  Returns 0, or -1.       */
int mxo_pack_blockwise(const float *W, int N, int K, int ldw, const uint8_t *table, const uint8_t *meta,
                       int16_t *q, uint8_t *zeros, uint16_t *scales)
{
    if (N < 0 || K <= 0 || K % MXO_BLK_COLS || ldw < K) return -1;
    for (int c = 0; c < 4; ++c)
        if (table[c] < 1 || table[c] > 8) return -1;
    const int KB = K / MXO_BLK_COLS;
    int8_t c8[MXO_BLK_COLS];
    uint8_t ca[MXO_BLK_COLS];
    for (int n = 0; n < N; ++n)
        for (int kb = 0; kb < KB; ++kb) {
            const float *w = W + (size_t)n * ldw + (size_t)kb * MXO_BLK_COLS;
            const int b = block_bits(meta, table, KB, n / MXO_BLK_ROWS, kb);
            int16_t *qo = q + (size_t)n * K + (size_t)kb * MXO_BLK_COLS;
            uint16_t sb;
            if (b == 8) {
                mxo_quant_sym8(w, MXO_BLK_COLS, c8, &sb);
                for (int k = 0; k < MXO_BLK_COLS; ++k) qo[k] = c8[k];
                zeros[(size_t)n * KB + kb] = 0;
            } else {
                uint8_t z;
                mxo_quant_asym(w, MXO_BLK_COLS, b, ca, &z, &sb);
                for (int k = 0; k < MXO_BLK_COLS; ++k) qo[k] = ca[k];
                zeros[(size_t)n * KB + kb] = z;
            }
            scales[(size_t)n * KB + kb] = sb;
        }
    return 0;
}

/* The two-step GEMM over a block-wise layer (MixLLM section 3.3 applied to  */
/* each 128-column group), fp64, at the listed (m, n) pairs (pairs == NULL: */
/* every (m, n), row-major [M][N]), two ways that must agree:               */
/*   Y_def = sum_k (Aq s_a)[m][k] * ((q - z) s_w)[n][k]                     */
/*   Y_two = sum_kb s_a[m] s_w[n][kb] P[m][n][kb],                          */
/*           P[m][n][kb] = sum_{k in kb} Aq[m][k] (q[n][k] - z[n][kb])       */
/* P (optional, [n_pairs][KB] int64) receives the partials.  s_a: one fp16   */
/* scale per token.  Returns the largest |P|, or -1 on bad arguments.       */
int64_t mxo_gemm_blockwise(const int8_t *Aq, const uint16_t *s_a, int M, int K, int N, const int16_t *q,
                           const uint8_t *zeros, const uint16_t *scales, const int32_t *pair_m,
                           const int32_t *pair_n, long n_pairs, double *Y_def, double *Y_two, int64_t *P)
{
    if (M < 0 || N < 0 || K <= 0 || K % MXO_BLK_COLS) return -1;
    const int KB = K / MXO_BLK_COLS;
    const long total = pair_m ? n_pairs : (long)M * N;
    int64_t pmax = 0;
    for (long t = 0; t < total; ++t) {
        const int m = pair_m ? pair_m[t] : (int)(t / (N > 0 ? N : 1));
        const int n = pair_m ? pair_n[t] : (int)(t % (N > 0 ? N : 1));
        if (m < 0 || m >= M || n < 0 || n >= N) return -1;
        const double sa = mxo_fp16_value(s_a[m]);
        double ydef = 0.0, ytwo = 0.0;
        for (int kb = 0; kb < KB; ++kb) {
            const double sw = mxo_fp16_value(scales[(size_t)n * KB + kb]);
            const int z = zeros[(size_t)n * KB + kb];
            int64_t p = 0;
            for (int k = kb * MXO_BLK_COLS; k < (kb + 1) * MXO_BLK_COLS; ++k) {
                const int a = Aq[(size_t)m * K + k];
                const int w = q[(size_t)n * K + k] - z;
                ydef += ((double)a * sa) * ((double)w * sw);
                p += (int64_t)a * (int64_t)w;
            }
            ytwo += sa * sw * (double)p;
            if (P) P[t * KB + kb] = p;
            if (llabs(p) > pmax) pmax = llabs(p);
        }
        Y_def[t] = ydef;
        Y_two[t] = ytwo;
    }
    return pmax;
}
