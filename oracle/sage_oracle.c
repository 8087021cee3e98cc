/*
 * sage_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of the SageAttention 8-bit
 * forward pass.  It exists so that the CUDA library can be checked against
 * something written straight from the method's description; nothing in the
 * product path may call it.  It shares no code, header or constant table with
 * the CUDA sources.
 *
 * Two results are computed from the same inputs:
 *
 *   R  the plain definition  softmax(QK^T * sm_scale) V  in fp64
 *      (page "Attention机制优化：从FlashAttention到SageAttention的工程实践",
 *       section 2.1 "数学原理与经典实现"), two-pass max-subtracted softmax;
 *
 *   E  a step-by-step emulation of the quantised method, in the order the
 *      SageAttention pages give it:
 *        - K smoothing: subtract the per-channel mean of K over the tokens
 *          (page "SageAttention v1/v2/v2++/v3" (dtcms.com), v1 bullet 1;
 *           page "SageAttention -- brand new attention" (postsniper.ru),
 *           "SageAttention" bullet 1);
 *        - per-block INT8 quantisation  delta = max|A|/127,  A^ = round(A/delta)
 *          (postsniper.ru page, quantisation intro steps 1-2; dtcms.com page,
 *           v1 item (1) "per-block");
 *        - INT8 QK^T, rescaled by deltaQ*deltaK (postsniper.ru page, step 3),
 *          the rescale fused with the softmax scale ("fuse scaling and
 *          unscaling with the neighbouring operations", postsniper.ru page,
 *          "SageAttention" bullet 2);
 *        - FlashAttention tiled online softmax (csdn/intelliparadigm page,
 *          section 3.1 "Online Softmax");
 *        - P.V in 16 bits (postsniper.ru page, "SageAttention" bullet 3) or
 *          P, V in FP8 with a two-level FP32 accumulation (dtcms.com page,
 *          SageAttention 2 bullets 1 and 3; postsniper.ru page,
 *          "SageAttention2" bullet 3).
 *
 * Where the pages leave an arithmetic detail open, the reading taken is stated
 * at the step.  Every fp32 step is a single IEEE-754 binary32 operation (the
 * file is compiled with -ffp-contract=off and without fast-math); fmaf() is
 * used only where a fused multiply-add is part of the stated step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_RANGE 1
#define ORACLE_ERR_ARG 2

/* ------------------------------------------------------------------------ */
/* Number formats.                                                           */
/* ------------------------------------------------------------------------ */

/*
 * Round x to the nearest value (ties to even) of a binary floating-point format
 * with `mant` stored mantissa bits and minimum normal exponent `emin`
 * (subnormals included).  Values beyond `maxval` saturate to +-maxval when
 * `saturate` is set, else become +-inf.  x must be finite.
 */
static double round_to_format(double x, int mant, int emin, double maxval, int saturate)
{
    if (x == 0.0) return x;
    if (isinf(x)) return saturate ? copysign(maxval, x) : x;
    int ex;
    (void)frexp(x, &ex);            /* |x| = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;                 /* exponent of the leading bit  */
    if (e < emin) e = emin;         /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, e - mant);
    double r = nearbyint(x / quantum) * quantum;   /* x/quantum is exact */
    if (fabs(r) > maxval) {
        if (saturate) r = copysign(maxval, x);
        else r = copysign(INFINITY, x);
    }
    return r;
}

/* IEEE binary16: 10 mantissa bits, emin -14, max 65504. */
double oracle_round_fp16(double x) { return round_to_format(x, 10, -14, 65504.0, 0); }

/* bfloat16: 7 mantissa bits, emin -126, max (2 - 2^-7) * 2^127. */
double oracle_round_bf16(double x)
{
    return round_to_format(x, 7, -126, ldexp(255.0, 120), 0);
}

/*
 * OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities, S.1111.111 is NaN, largest finite 448, smallest
 * subnormal 2^-9.  Encoding rounds to nearest-even and saturates finite
 * values beyond 448 to +-448 (the "satfinite" behaviour).
 */
uint8_t oracle_e4m3_encode(float xf)
{
    double x = (double)xf;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x)) return 0x7F;
    double r = fabs(round_to_format(fabs(x), 3, -6, 448.0, 1));
    if (r == 0.0) return sign;
    int ex;
    double f = frexp(r, &ex);       /* r = f * 2^ex */
    int e = ex - 1;
    if (e < -6) {                   /* subnormal: r = m * 2^-9 */
        int m = (int)(r * 512.0);
        return (uint8_t)(sign | m);
    }
    int m = (int)((f * 2.0 - 1.0) * 8.0);   /* 3-bit fraction */
    return (uint8_t)(sign | ((e + 7) << 3) | m);
}

double oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* Step A1: K channel mean.                                                  */
/* ------------------------------------------------------------------------ */

/*
 * Mean of K over the n tokens of one (sequence, head), per channel.
 *
 * The pages say only "subtract the mean" (dtcms.com page, v1 bullet 1).  The
 * codes that follow depend on every bit of the mean, so the mean is defined
 * so that its value does not depend on summation order: each element is put
 * on the fixed-point grid 2^-24 (round half to even; exact for every fp16
 * value, and for every bf16 value of magnitude >= 2^-24), the grid integers
 * are summed exactly in int64, and the sum is divided once in fp64 and
 * rounded to fp32:  m_d = fp32( fp64(S_d) / (n * 2^24) ).
 *
 * Range: |k| < 2^16 keeps every partial sum inside int64 for n < 2^23.
 * Returns ORACLE_ERR_RANGE for a non-finite or too-large element.
 *
 * k: row t of the head at k + t*ld, D channels.  sum_out, mean_out: [D].
 */
int oracle_k_mean(const float* k, long n, int D, long ld, int64_t* sum_out, float* mean_out)
{
    int status = ORACLE_OK;
    for (int d = 0; d < D; ++d) {
        int64_t s = 0;
        for (long t = 0; t < n; ++t) {
            double x = (double)k[t * ld + d];
            if (!(fabs(x) < 65536.0)) { status = ORACLE_ERR_RANGE; continue; }
            s += (int64_t)nearbyint(x * 16777216.0);
        }
        sum_out[d] = s;
        mean_out[d] = (float)((double)s / ((double)n * 16777216.0));
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* Steps A2/A3: per-block INT8 quantiser.                                    */
/* ------------------------------------------------------------------------ */

/*
 * Quantise one block of `rows` tokens x D channels (the block is the
 * "per-block" granularity; its token count is a parameter, 128 here).
 *
 * postsniper.ru page, quantisation intro:
 *   step 1  delta = max|A| / 127
 *   step 2  A^ = round(A / delta)
 * Readings: the division by delta is carried out as a multiplication by the
 * block constant s = 127/max|A| (one fp32 division per block, one fp32
 * multiplication per element); "round" is round-half-to-even; codes are
 * clamped to [-127, 127]; a block whose max|A| is 0 gets delta = 0 and all
 * codes 0.  For K, the element is first smoothed, x = fp32(k - m_d).
 *
 * x: row r at x + r*ld.  mean: per-channel mean to subtract, or NULL.
 * codes: [rows][D] int8.  Returns delta.
 */
float oracle_quant_block(const float* x, int rows, int D, long ld, const float* mean,
                         int8_t* codes)
{
    float amax = 0.0f;
    for (int r = 0; r < rows; ++r)
        for (int d = 0; d < D; ++d) {
            float y = x[r * ld + d];
            if (mean) y = y - mean[d];
            float a = fabsf(y);
            if (a > amax) amax = a;
        }
    if (amax == 0.0f) {
        memset(codes, 0, (size_t)rows * D);
        return 0.0f;
    }
    float delta = amax / 127.0f;
    float s = 127.0f / amax;
    for (int r = 0; r < rows; ++r)
        for (int d = 0; d < D; ++d) {
            float y = x[r * ld + d];
            if (mean) y = y - mean[d];
            float c = nearbyintf(y * s);
            if (c > 127.0f) c = 127.0f;
            if (c < -127.0f) c = -127.0f;
            codes[r * D + d] = (int8_t)c;
        }
    return delta;
}

/*
 * Quantise all blocks of one (sequence, head): n tokens in blocks of `blk`
 * tokens; the last block may be partial.  codes: [nblk*blk][D], rows past n
 * are written as 0 (padding); delta: [nblk].
 */
void oracle_quant_head(const float* x, long n, int D, long ld, const float* mean, int blk,
                       int8_t* codes, float* delta)
{
    long nblk = (n + blk - 1) / blk;
    memset(codes, 0, (size_t)nblk * blk * D);
    for (long b = 0; b < nblk; ++b) {
        long r0 = b * blk;
        int rows = (int)((n - r0) < blk ? (n - r0) : blk);
        delta[b] = oracle_quant_block(x + r0 * ld, rows, D, ld, mean, codes + r0 * D);
    }
}

/* ------------------------------------------------------------------------ */
/* Step A4: V to FP8 (E4M3), per channel.                                    */
/* ------------------------------------------------------------------------ */

/*
 * dtcms.com page, SageAttention 2 bullet 1 ("quantise (P, V) to FP8").
 * Readings: format E4M3; one scale per channel over the n tokens (a per-token
 * V scale would not factor out of sum_t P_t V_t, a per-channel one does, by
 * the same argument as step 3 of the postsniper.ru quantisation intro);
 * deltaV_d = max_t|v_td| / 448, codes = e4m3(v * (448 / max|v|)).
 *
 * codes: [n][D] e4m3 bytes.  delta: [D].
 */
void oracle_quant_v_fp8(const float* v, long n, int D, long ld, uint8_t* codes, float* delta)
{
    for (int d = 0; d < D; ++d) {
        float amax = 0.0f;
        for (long t = 0; t < n; ++t) {
            float a = fabsf(v[t * ld + d]);
            if (a > amax) amax = a;
        }
        float s = 0.0f;
        if (amax > 0.0f) {
            delta[d] = amax / 448.0f;
            s = 448.0f / amax;
        } else {
            delta[d] = 0.0f;
        }
        for (long t = 0; t < n; ++t) codes[t * D + d] = oracle_e4m3_encode(v[t * ld + d] * s);
    }
}

/* ------------------------------------------------------------------------ */
/* Step A5: INT8 QK^T, exact.                                                */
/* ------------------------------------------------------------------------ */

/* S[i][j] = sum_d qc[i][d] * kc[j][d] for rows i0..i0+mi-1, keys j0..j0+nj-1. */
void oracle_qk_int(const int8_t* qc, const int8_t* kc, int D, long i0, int mi, long j0, int nj,
                   int32_t* S)
{
    for (int i = 0; i < mi; ++i)
        for (int j = 0; j < nj; ++j) {
            int32_t acc = 0;
            for (int d = 0; d < D; ++d)
                acc += (int32_t)qc[(i0 + i) * D + d] * (int32_t)kc[(j0 + j) * D + d];
            S[i * nj + j] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* R: the plain definition, fp64.                                            */
/* ------------------------------------------------------------------------ */

/*
 * out_i = sum_j softmax_j(sm_scale * q_i . k_j) v_j over j < n (j <= i when
 * causal, top-left aligned), for the listed rows of one (sequence, head).
 * Two-pass softmax with the row maximum subtracted.  out: [nrows][D], fp64.
 */
void oracle_attn_ref_rows(const float* q, const float* k, const float* v, long n, int D,
                          long ldq, long ldk, long ldv, double sm_scale, int causal,
                          const long* rows, long nrows, double* out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        long jn = causal ? i + 1 : n;
        double* logit = (double*)malloc(sizeof(double) * (size_t)jn);
        double mx = -INFINITY;
        for (long j = 0; j < jn; ++j) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += (double)q[i * ldq + d] * (double)k[j * ldk + d];
            logit[j] = acc * sm_scale;
            if (logit[j] > mx) mx = logit[j];
        }
        double denom = 0.0;
        double* o = out + r * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (long j = 0; j < jn; ++j) {
            double w = exp(logit[j] - mx);
            denom += w;
            for (int d = 0; d < D; ++d) o[d] += w * (double)v[j * ldv + d];
        }
        for (int d = 0; d < D; ++d) o[d] /= denom;
        free(logit);
    }
}

/* ------------------------------------------------------------------------ */
/* E: the quantised method, step by step.                                    */
/* ------------------------------------------------------------------------ */

/* fp32(log2 448): the FP8 P scale when it is applied in the exponent */
#define LOG2_448F 8.807354927062988f

/*
 * Emulated output rows of one (sequence, head).
 *
 * Inputs are the outputs of the steps above: q codes/deltas, k codes/deltas
 * (smoothed K), and either the 16-bit V values (pv_mode 0) or V's E4M3 codes
 * and per-channel deltas (pv_mode 1).  `blk` is the quantisation block; `kv`
 * (a divisor of blk) is the key-tile length of the tiled online softmax and of
 * the FP8 two-level flush.  kappa = fp32(sm_scale * log2(e)): the softmax
 * runs in base 2.
 *
 * THE METHOD (the plain form; kv = blk = 128, tau = 0, p8_exp = 0).  The
 * pages give FlashAttention's tiled online softmax ("Attention机制优化",
 * section 3.1) over the key blocks of the quantised K, and flush the FP8
 * partial sums into the fp32 accumulator once per block ("SageAttention
 * v1/v2/v2++/v3" overview, SageAttention 2 bullet 3).  For each row i (query
 * block I = i / blk) and key tile T = 0, 1, ... in ascending order (tiles
 * starting at or before i when causal), the tile's keys lying in quantisation
 * block J = T*kv / blk, with m = -inf, l = 0, O = 0:
 *
 *   S_ij   = sum_d q^_id k^_jd                       exact int32
 *   c_IJ   = fp32( fp32(deltaQ_I * deltaK_J) * kappa )   dequant x softmax scale
 *   mb     = fp32(max_j S_ij * c_IJ)                   the tile's scaled max
 *   m_new  = max(m, mb)                                the running maximum
 *   arg_ij = fmaf(S_ij, c_IJ, -m_new)                 dequant, scale and max
 *                                                     subtraction in one fused
 *                                                     multiply-add (reading of
 *                                                     "fuse scaling/unscaling
 *                                                     with neighbouring ops")
 *   p_ij   = fp32(2^arg_ij)                           (2^x evaluated in fp64)
 *   alpha  = fp32(2^fp32(m - m_new))
 *   l      = fp32(fp32(alpha * l) + fp32(sum_j p_ij))  (FlashAttention normaliser,
 *                                                     of the unquantised p)
 *   pv_mode 0 (16-bit P.V):
 *     P_ij  = p_ij rounded to V's 16-bit format
 *     Part  = fp32(sum_j P_ij v_jd)                   (products summed in fp64)
 *     O_d   = fp32(fp32(alpha * O_d) + Part_d)
 *   pv_mode 1 (FP8 P.V, two-level accumulation; static P scale 448, since
 *   p <= 1 at the running maximum):
 *     P^_ij = e4m3(fp32(p_ij * 448))
 *     Part  = fp32(sum_j dec(P^_ij) dec(v^_jd))       one key tile's partial
 *     O_d   = fp32(fp32(alpha * O_d) + Part_d)        flushed into the fp32
 *                                                     accumulator every tile
 *   m = m_new
 *
 * Finally out_d = fp32(O_d / l)   (pv_mode 0), or
 *           out_d = fp32(O_d * deltaV_d / (448 l))   (pv_mode 1; the exact
 *           value of the expression, rounded once).
 *
 * Masked keys (j >= n, or j > i when causal) take no part in the maximum and
 * contribute p = 0.  (A tile is entered only if it holds at least one
 * unmasked key of the row.)
 *
 * OTHER EVALUATION ORDERS of the same method.  In exact arithmetic the
 * rescale factors cancel in O / l, so the following change only roundings;
 * they exist so that a faster evaluation order can also be checked step for
 * step:
 *   kv < blk   shorter key tiles (both parts of a block share its deltas);
 *   tau > 0    the maximum in use moves only when the tile's maximum exceeds
 *              it by more than tau (base 2): m_new = mb if mb > m + tau,
 *              else m; p may then reach 2^tau (16-bit P.V only: FP8 needs
 *              p <= 1);
 *   p8_exp = 1 (FP8 P.V) the P scale is applied in the exponent: arg_ij =
 *              fmaf(S_ij, c_IJ, fp32(L - m_new)), L = fp32(log2 448), so p_ij
 *              = 448 2^(t - m) directly, P^_ij = e4m3(p_ij), l sums these
 *              scaled p, the flush is O_d = fmaf(alpha, O_d, Part_d), and
 *              out_d = fp32(fp32(O_d * deltaV_d) / l) (the 448 of P and of l
 *              cancel).
 *
 * p16_format: 0 = fp16, 1 = bf16 (V's own format, used for P in pv_mode 0).
 * out: [nrows][D] fp32.
 *
 * per_token = 1: the other quantisation granularity of the dtcms.com page
 * (SageAttention v1 item (1): "per-block or per-token"; the postsniper.ru
 * post quantises "each row separately"): qdelta[i] and kdelta[j] are one delta
 * per token, and the dequantisation is taken key first, then query:
 *   y_ij   = fp32(S_ij * deltaK_j)
 *   c_i    = fp32(deltaQ_i * kappa)
 *   mb     = fp32(max_j y_ij * c_i)
 *   arg_ij = fmaf(y_ij, c_i, -m_new)
 * (the product (A^ B^) deltaA deltaB of the quantisation intro, step 3, with a
 * per-row deltaA and a per-column deltaB); everything else as above.
 *
 * bk != NULL: Q smoothing (SageAttention2, dtcms.com page, v2 bullet 2, and
 * the postsniper.ru post's SageAttention2 bullet 1, which also normalise Q).
 * The Q codes are those of q~ = q - qmean_I (per-block channel mean of Q), and
 * the part of q.k~ that the mean carries is added back per key:
 * bk[I*ldb + j] = kappa * qmean_I . k~_j (see oracle_q_smooth_bias).
 * Per-block deltas only:
 *   c_IJ   = fp32( fp32(deltaQ_I * deltaK_J) * kappa )
 *   y_ij   = fmaf(S_ij, c_IJ, bk_Ij)                  scaled logit
 *   mb     = max_j y_ij
 *   arg_ij = fp32(y_ij - m_new)    (p8_exp: fp32(y_ij + fp32(L - m_new)))
 * everything else as above.
 */
void oracle_attn_emul_rows(const int8_t* qc, const float* qdelta, const int8_t* kc,
                           const float* kdelta, const float* v, long ldv, const uint8_t* vc,
                           const float* vdelta, long n, int D, int blk, int kv, float kappa,
                           float tau, int causal, int pv_mode, int p16_format, const long* rows,
                           long nrows, float* out, int per_token, const float* bk, long ldb,
                           int p8_exp)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < nrows; ++r) {
        long i = rows[r];
        long I = i / blk;
        long ntile = (n + kv - 1) / kv;
        long Tend = causal ? i / kv + 1 : ntile;
        float m = -INFINITY, l = 0.0f;
        float* O = (float*)calloc((size_t)D, sizeof(float));
        double* part = (double*)malloc(sizeof(double) * (size_t)D);
        int32_t* S = (int32_t*)malloc(sizeof(int32_t) * (size_t)kv);
        float* p = (float*)malloc(sizeof(float) * (size_t)kv);
        float* y = (float*)malloc(sizeof(float) * (size_t)kv);
        for (long T = 0; T < Tend; ++T) {
            long j0 = T * kv;
            long J = j0 / blk;
            long j1 = j0 + kv < n ? j0 + kv : n;
            if (causal && j1 > i + 1) j1 = i + 1;
            int nj = (int)(j1 - j0);
            int32_t smax = INT32_MIN;
            for (int jj = 0; jj < nj; ++jj) {
                int32_t acc = 0;
                for (int d = 0; d < D; ++d)
                    acc += (int32_t)qc[i * D + d] * (int32_t)kc[(j0 + jj) * D + d];
                S[jj] = acc;
                if (acc > smax) smax = acc;
            }
            float c, mblk;
            if (bk) {
                /* Q smoothing: the per-key mean term joins before the maximum */
                const float* bI = bk + I * ldb + j0;
                c = (qdelta[I] * kdelta[J]) * kappa;
                float ymax = -INFINITY;
                for (int jj = 0; jj < nj; ++jj) {
                    y[jj] = fmaf((float)S[jj], c, bI[jj]);
                    if (y[jj] > ymax) ymax = y[jj];
                }
                mblk = ymax;
            } else if (!per_token) {
                /* one delta per 128-token block of Q and of K */
                c = (qdelta[I] * kdelta[J]) * kappa;
                mblk = (float)smax * c;
            } else {
                /* one delta per token: S_ij deltaK_j first (a key's own
                 * scale), then the query row's deltaQ_i kappa */
                c = qdelta[i] * kappa;
                float ymax = -INFINITY;
                for (int jj = 0; jj < nj; ++jj) {
                    y[jj] = (float)S[jj] * kdelta[j0 + jj];
                    if (y[jj] > ymax) ymax = y[jj];
                }
                mblk = ymax * c;
            }
            float m_new = mblk > m + tau ? mblk : m;
            float alpha = (float)exp2((double)(m - m_new));
            /* p8_exp: p is formed already scaled by 448, as 2^(arg + log2 448) */
            const int fold = pv_mode == 1 && p8_exp;
            const float sub = fold ? LOG2_448F - m_new : -m_new;
            double psum = 0.0;
            for (int jj = 0; jj < nj; ++jj) {
                float arg = bk ? y[jj] + sub
                            : per_token ? fmaf(y[jj], c, sub) : fmaf((float)S[jj], c, sub);
                p[jj] = (float)exp2((double)arg);
                psum += (double)p[jj];
            }
            l = alpha * l + (float)psum;
            for (int d = 0; d < D; ++d) part[d] = 0.0;
            if (pv_mode == 0) {
                for (int jj = 0; jj < nj; ++jj) {
                    double P = p16_format ? oracle_round_bf16(p[jj]) : oracle_round_fp16(p[jj]);
                    const float* vr = v + (j0 + jj) * ldv;
                    for (int d = 0; d < D; ++d) part[d] += P * (double)vr[d];
                }
                for (int d = 0; d < D; ++d) O[d] = alpha * O[d] + (float)part[d];
            } else {
                for (int jj = 0; jj < nj; ++jj) {
                    const float p448 = fold ? p[jj] : p[jj] * 448.0f;
                    double P = oracle_e4m3_decode(oracle_e4m3_encode(p448));
                    const uint8_t* vr = vc + (j0 + jj) * D;
                    for (int d = 0; d < D; ++d) part[d] += P * oracle_e4m3_decode(vr[d]);
                }
                for (int d = 0; d < D; ++d)
                    O[d] = fold ? fmaf(alpha, O[d], (float)part[d]) : alpha * O[d] + (float)part[d];
            }
            m = m_new;
        }
        float* o = out + r * D;
        for (int d = 0; d < D; ++d) {
            if (pv_mode == 0) o[d] = O[d] / l;
            else if (p8_exp) o[d] = (O[d] * vdelta[d]) / l;  /* the 448 of P and of l cancel */
            else o[d] = (float)((double)O[d] * (double)vdelta[d] / (448.0 * (double)l));
        }
        free(O); free(part); free(S); free(p); free(y);
    }
}

/* ------------------------------------------------------------------------ */
/* Q smoothing: the per-key term of the block mean.                          */
/* ------------------------------------------------------------------------ */

/*
 * With q = q~ + qmean_I for the rows of query block I (SageAttention2's
 * smoothing of Q, dtcms.com page, v2 bullet 2), the smoothed logit splits as
 *   q . k~_j = q~ . k~_j + qmean_I . k~_j,
 * the first part quantised like any Q block, the second a dot product that
 * depends on the block and the key only.  (qmean_I . m, the part through the
 * K mean, is a constant per row and leaves the softmax unchanged, as for K
 * smoothing; the term here uses the smoothed k~ = fp32(k - kmean) that the K
 * codes come from.)
 *
 * The pages fix no precision for this dot product.  The plain form:
 *   out[I*ldo + j] = fp32( kappa * sum_d qmean[I][d] * k~_j[d] )
 * with the products and the sum in fp64 (exact products of fp32 values) and
 * one rounding at the end.
 *
 * qmean: [nb][D]; k: row j at k + j*ld; kmean: [D]; out: [nb][ldo], columns
 * j < n written.
 */
void oracle_q_smooth_bias(const float* qmean, long nb, const float* k, long n, int D, long ld,
                          const float* kmean, float kappa, float* out, long ldo)
{
    for (long I = 0; I < nb; ++I) {
        for (long j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) {
                const float ks = k[j * ld + d] - kmean[d];
                acc += (double)qmean[I * D + d] * (double)ks;
            }
            out[I * ldo + j] = (float)((double)kappa * acc);
        }
    }
}

/*
 * The same term in a fixed fp32 evaluation order (another evaluation order of
 * the step above, used to check such an order step for step):
 *   acc = 0;  acc = fmaf(qmean[I][d], k~_j[d], acc)  for d = 0 .. D-1
 *   out[I*ldo + j] = fp32(acc * kappa)
 */
void oracle_q_smooth_bias_fma(const float* qmean, long nb, const float* k, long n, int D, long ld,
                              const float* kmean, float kappa, float* out, long ldo)
{
    for (long I = 0; I < nb; ++I) {
        for (long j = 0; j < n; ++j) {
            float acc = 0.0f;
            for (int d = 0; d < D; ++d) {
                const float ks = k[j * ld + d] - kmean[d];
                acc = fmaf(qmean[I * D + d], ks, acc);
            }
            out[I * ldo + j] = acc * kappa;
        }
    }
}
