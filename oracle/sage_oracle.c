/*
 * Plain CPU oracle for the SageAttention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls this
 * file: only the tests, the package's smoke check and the CPU-baseline leg of the
 * benchmark do. It shares no code, header, table or constant generator with the CUDA
 * library.
 *
 * What it restates, with the passage each step follows:
 *   - Smooth K: K <- K - mean(K), the mean taken per channel over the tokens of one
 *     head. (「SageAttention：低比特量化Attention，实现推理加速」, section "技术方案", paragraph "对 K 进行平滑处理".)
 *   - Per-block INT8 quantization of Q and K, one fp32 scale per block of tokens of
 *     FlashAttention block size; INT8 products accumulate in INT32. (Same section,
 *     paragraph "对 Q, K 进行分块 INT8 量化".) The scale is amax/127 (the method's
 *     INT8 symmetric range); Q blocks are 128 tokens, K blocks 64 tokens.
 *   - FlashAttention tiling with online softmax over KV tiles; P and V in FP16 for
 *     P.V. (Same section, paragraph "对 P, V 采用 FP16 数据类型的矩阵乘法累加器".)
 *   - FP8 mode: P and V quantized to E4M3, each tile's P.V product summed into an
 *     FP32-or-wider accumulator across tiles. (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, section
 *     "技术方案", items (3) and (4).)
 *   - Smooth V (FP8 mode): V <- V - mean(V) with the mean per channel over the tokens
 *     of one head, the attention run on the smoothed V, and mean(V) added to the
 *     output. (Same section, the paragraph after item (4).)
 *   - Smooth Q: Q <- Q - mean(Q) (per channel over the query tokens of one head) before
 *     quantizing, and the vector-matrix product mean(Q) K^T added back to the scores.
 *     (Same section, item (1).)
 *   - The exact reference O = softmax(sm_scale Q K^T + mask) V in fp64, and the
 *     smoothing invariant softmax(QK^T) = softmax(Q(K - mean K)^T) it must satisfy.
 *
 * Precision: the pages fix fp32 block scales, INT8 codes with INT32 products, FP16
 * P/V and E4M3 P/V; every other quantity (the K-mean sum, dequantized scores, the
 * exponentials, the row sums and the output accumulator) is computed here in fp64.
 * Every function is one head at a time with an explicit row stride, so the same code
 * serves the dense [B,H,N,d] layout and the packed varlen [T,H,d] layout.
 *
 * Parity of the quantized attention as a whole is pinned by its special cases and
 * by the fp64 attention (no page prints a numeric example).
 */
#include <stdint.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- number formats */

/* IEEE binary16 bits -> exact value. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);    /* (1024+m) * 2^(e-15-10) */
    return sign ? -v : v;
}

/* Round a real to the nearest binary16 value, ties to even; overflow to +-inf. */
double oracle_round_f16(double x)
{
    if (isnan(x) || isinf(x) || x == 0.0)
        return x;
    double a = fabs(x);
    int E;
    frexp(a, &E);               /* a = f * 2^E with f in [0.5, 1): unbiased exponent E-1 */
    int ue = E - 1;
    if (ue < -14)
        ue = -14;               /* subnormal range shares the quantum 2^-24 */
    double quantum = ldexp(1.0, ue - 10);
    double r = nearbyint(a / quantum) * quantum;    /* exact: division by a power of two */
    if (r > 65504.0)
        r = INFINITY;           /* |x| >= 65520 rounds past the largest finite value */
    return x < 0 ? -r : r;
}

/* Exact binary16 value -> its bit pattern (the value must be representable). */
uint16_t oracle_f16_bits(double v)
{
    uint16_t sign = (v < 0 || (v == 0 && signbit(v))) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return 0x7e00;
    if (isinf(v))
        return sign | 0x7c00;
    if (a == 0)
        return sign;
    if (a < ldexp(1.0, -14))
        return sign | (uint16_t)(a / ldexp(1.0, -24));
    int E;
    double f = frexp(a, &E);    /* a = f * 2^E, f in [0.5,1) */
    int e = E - 1 + 15;
    uint16_t m = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(e << 10) | m;
}

/* OCP FP8 E4M3 (the "fn" variant: bias 7, no infinities, max finite 448) -> value. */
double oracle_e4m3_to_f64(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xf;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);                  /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);        /* (1+m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Round a real to E4M3, ties to even, saturating to +-448 ("satfinite"). Returns bits. */
uint8_t oracle_e4m3_encode(double x)
{
    if (isnan(x))
        return 0x7f;
    uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? 0x80 : 0;
    double a = fabs(x);
    if (a == 0)
        return sign;
    double r;
    if (a >= 448.0) {
        r = 448.0;
    } else {
        int E;
        frexp(a, &E);
        int ue = E - 1;
        if (ue < -6)
            ue = -6;            /* subnormals share the quantum 2^-9 */
        double quantum = ldexp(1.0, ue - 3);
        r = nearbyint(a / quantum) * quantum;
        if (r > 448.0)
            r = 448.0;          /* 464 and above would round to 480: saturate */
    }
    /* value -> bits */
    if (r < ldexp(1.0, -6))
        return sign | (uint8_t)(r / ldexp(1.0, -9));
    int E;
    double f = frexp(r, &E);
    int e = E - 1 + 7;
    uint8_t m = (uint8_t)((f * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(e << 3) | m;
}

/* ------------------------------------------- smooth K and V: per-channel token mean */

/*
 * mu[c] = (sum over the n tokens of X[t, c]) / n, summed in fp64 in token order, the
 * quotient taken in fp64 and rounded once to fp32. One head; row t of channel c is at
 * X[t*stride + c]. X is K for smooth K and V for smooth V.
 */
void oracle_head_channel_mean(const uint16_t *X, int64_t n, int64_t stride, int d, float *mu)
{
    for (int c = 0; c < d; c++) {
        double s = 0.0;
        for (int64_t t = 0; t < n; t++)
            s += oracle_f16_to_f64(X[t * stride + c]);
        mu[c] = n > 0 ? (float)(s / (double)n) : 0.0f;
    }
}

/* ------------------------------------------------------ per-block INT8 quantization */

/*
 * Blocks of `blk` consecutive tokens of one head (the last one ragged: only its valid
 * rows enter the scale). Element x = fp32(X[t,c]) - mu[c] (one fp32 subtraction; mu may
 * be NULL for "no smoothing"). scale = amax / 127 in fp32; code = round-half-even(x /
 * scale) in fp32, clamped to [-127, 127]; an all-zero block gets scale 0 and codes 0.
 * codes use the same row stride as X; scales[b] for block b.
 */
void oracle_head_quant_int8(const uint16_t *X, const float *mu, int64_t n, int64_t stride,
                            int d, int blk, int8_t *codes, float *scales)
{
    int64_t nblk = (n + blk - 1) / blk;
    for (int64_t b = 0; b < nblk; b++) {
        int64_t t0 = b * blk, t1 = t0 + blk < n ? t0 + blk : n;
        float amax = 0.0f;
        for (int64_t t = t0; t < t1; t++)
            for (int c = 0; c < d; c++) {
                float x = (float)oracle_f16_to_f64(X[t * stride + c]);
                if (mu)
                    x = x - mu[c];
                float a = fabsf(x);
                if (a > amax)
                    amax = a;
            }
        float s = amax / 127.0f;
        scales[b] = s;
        for (int64_t t = t0; t < t1; t++)
            for (int c = 0; c < d; c++) {
                float x = (float)oracle_f16_to_f64(X[t * stride + c]);
                if (mu)
                    x = x - mu[c];
                int code = 0;
                if (s != 0.0f) {
                    float q = x / s;
                    double r = nearbyint((double)q);     /* ties to even */
                    if (r > 127)
                        r = 127;
                    if (r < -127)
                        r = -127;
                    code = (int)r;
                }
                codes[t * stride + c] = (int8_t)code;
            }
    }
}

/*
 * V to E4M3 with one fp32 scale per channel over all tokens of the head. Element
 * x = fp32(V[t,c]) - mu[c] (one fp32 subtraction; mu is the channel mean of V for
 * smooth V, NULL for none); s[c] = amax_t |x| / 448; code = e4m3_rne_satfinite(x / s[c])
 * with the quotient in fp32. A channel whose x are all zero gets scale 0 and codes 0.
 */
void oracle_head_quant_v_fp8(const uint16_t *V, const float *mu, int64_t n, int64_t stride,
                             int d, uint8_t *codes, float *scales)
{
    for (int c = 0; c < d; c++) {
        float amax = 0.0f;
        for (int64_t t = 0; t < n; t++) {
            float x = (float)oracle_f16_to_f64(V[t * stride + c]);
            if (mu)
                x = x - mu[c];
            float a = fabsf(x);
            if (a > amax)
                amax = a;
        }
        float s = amax / 448.0f;
        scales[c] = s;
        for (int64_t t = 0; t < n; t++) {
            float x = (float)oracle_f16_to_f64(V[t * stride + c]);
            if (mu)
                x = x - mu[c];
            codes[t * stride + c] = (s != 0.0f) ? oracle_e4m3_encode((double)(x / s)) : 0;
        }
    }
}

/* ------------------------------------------------ smooth Q: score compensation */

/*
 * comp[j] = sum over c of muq[c] * (fp32(K[j,c]) - muk[c]) for the n keys of one head:
 * the mean(Q) K^T term that smoothing Q removes from the scores, with K as it enters
 * the INT8 quantization (smoothed by muk when that is not NULL, one fp32 subtraction).
 * The sum is taken in fp64 and rounded once to fp32.
 */
void oracle_head_q_comp(const uint16_t *K, const float *muk, const float *muq, int64_t n,
                        int64_t stride, int d, float *comp)
{
    for (int64_t j = 0; j < n; j++) {
        double acc = 0.0;
        for (int c = 0; c < d; c++) {
            float x = (float)oracle_f16_to_f64(K[j * stride + c]);
            if (muk)
                x = x - muk[c];
            acc += (double)muq[c] * (double)x;
        }
        comp[j] = (float)acc;
    }
}

/* ----------------------------------------------------------- quantized attention */

enum { ORACLE_PV_FP16 = 0, ORACLE_PV_FP8 = 1 };

/*
 * Quantized attention for query rows [r0, r1) of one head with nq queries and nk keys
 * (nq = nk for self-attention; nq < nk for queries that are the last nq positions of a
 * longer sequence, e.g. prefill against cached keys), following the method's steps in
 * order:
 *   S_int[i,j] = sum_c q[i,c] k[j,c] in integers (INT32 range is never exceeded);
 *   t[i,j] = (S_int * sq[i/qg] * sk[j/kg] + comp[j]) * sm_scale * log2(e) (base-2
 *   logits), where qg and kg are the tokens per Q and K scale (128 and 64 for per-block
 *   scales, 1 and 32 for the finer groups) and comp is the smooth-Q compensation
 *   (NULL: none);
 *   causal: key j is visible to query i when j <= i + (nk - nq) (the mask aligned at
 *   the bottom-right corner; the square mask j <= i when nq = nk); a query that sees no
 *   key (only when nq > nk) gets a zero output row;
 *   online softmax over KV tiles [j0, j0+tile_n) in ascending order, all in fp64:
 *     m' = max(m, max_j t), alpha = 2^(m - m') (0 when m = -inf),
 *     p_j = 2^(t_j - m'),  l = alpha l + sum p_j,
 *     FP16 mode: P_j = f16(p_j),          O = alpha O + sum_j P_j V[j]
 *     FP8 mode:  P_j = e4m3(448 p_j),     O = alpha O + sum_j P_j e4m3val(vc[j]);
 *   output row: FP16 mode O / l; FP8 mode O vs[c] / (448 l) + vm[c] (vm = the channel
 *   mean of V under smooth V, NULL for none); rounded to fp16.
 * `v` is fp16 bits (FP16 mode) or E4M3 codes (FP8 mode), row stride `stride`;
 * outputs are fp16 bits written at out[i*stride + c].
 */
void oracle_head_attn_quant(const int8_t *qc, const float *qs, const int8_t *kc,
                            const float *ks, const void *v, const float *vs, const float *vm,
                            const float *comp, int64_t nq, int64_t nk, int64_t stride, int d,
                            int causal,
                            int pv_mode, double sm_scale, int tile_n, int qg, int kg,
                            int64_t r0, int64_t r1, uint16_t *out)
{
    const double log2e = 1.4426950408889634073599246810019;   /* 1/ln 2 */
    if (r1 > nq)
        r1 = nq;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = r0; i < r1; i++) {
        double *O = (double *)calloc((size_t)d, sizeof(double));
        double *t = (double *)malloc((size_t)tile_n * sizeof(double));
        double m = -INFINITY, l = 0.0;
        int64_t jend = causal ? i + 1 + (nk - nq) : nk;  /* keys j < jend are visible */
        if (jend > nk)
            jend = nk;
        if (jend <= 0) {                                  /* no visible key: zero row */
            for (int c = 0; c < d; c++)
                out[i * stride + c] = 0;
            free(O);
            free(t);
            continue;
        }
        for (int64_t j0 = 0; j0 < jend; j0 += tile_n) {
            int64_t j1 = j0 + tile_n < jend ? j0 + tile_n : jend;
            double tmax = -INFINITY;
            for (int64_t j = j0; j < j1; j++) {
                int32_t S = 0;
                for (int c = 0; c < d; c++)
                    S += (int32_t)qc[i * stride + c] * (int32_t)kc[j * stride + c];
                double sij = (double)S * (double)qs[i / qg] * (double)ks[j / kg];
                if (comp)
                    sij += (double)comp[j];
                t[j - j0] = sij * sm_scale * log2e;
                if (t[j - j0] > tmax)
                    tmax = t[j - j0];
            }
            double mnew = m > tmax ? m : tmax;
            double alpha = (m == -INFINITY) ? 0.0 : exp2(m - mnew);
            l *= alpha;
            for (int c = 0; c < d; c++)
                O[c] *= alpha;
            for (int64_t j = j0; j < j1; j++) {
                double p = exp2(t[j - j0] - mnew);
                l += p;
                if (pv_mode == ORACLE_PV_FP16) {
                    double P = oracle_round_f16(p);
                    const uint16_t *vh = (const uint16_t *)v;
                    for (int c = 0; c < d; c++)
                        O[c] += P * oracle_f16_to_f64(vh[j * stride + c]);
                } else {
                    double P = oracle_e4m3_to_f64(oracle_e4m3_encode(448.0 * p));
                    const uint8_t *v8 = (const uint8_t *)v;
                    for (int c = 0; c < d; c++)
                        O[c] += P * oracle_e4m3_to_f64(v8[j * stride + c]);
                }
            }
            m = mnew;
        }
        for (int c = 0; c < d; c++) {
            double o = (pv_mode == ORACLE_PV_FP16) ? O[c] / l : O[c] * (double)vs[c] / (448.0 * l);
            if (pv_mode == ORACLE_PV_FP8 && vm)
                o += (double)vm[c];
            out[i * stride + c] = oracle_f16_bits(oracle_round_f16(o));
        }
        free(O);
        free(t);
    }
}

/* ---------------------------------------------------------------- exact attention */

/*
 * O = softmax(sm_scale Q K^T + causal mask) V for rows [r0, r1) of one head with nq
 * queries and nk keys, all in fp64 (two passes: row max, then normalized weights); the
 * causal mask is the bottom-right one of oracle_head_attn_quant, and a query with no
 * visible key gets a zero row. Inputs are fp64 so the smoothing invariant can be
 * checked with K - mean(K) exactly. Output at out[i*stride + c].
 */
void oracle_head_attn_fp64(const double *Q, const double *K, const double *V, int64_t nq,
                           int64_t nk, int64_t stride, int d, int causal, double sm_scale,
                           int64_t r0, int64_t r1, double *out)
{
    if (r1 > nq)
        r1 = nq;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = r0; i < r1; i++) {
        int64_t jend = causal ? i + 1 + (nk - nq) : nk;
        if (jend > nk)
            jend = nk;
        if (jend <= 0) {
            for (int c = 0; c < d; c++)
                out[i * stride + c] = 0.0;
            continue;
        }
        double *s = (double *)malloc((size_t)jend * sizeof(double));
        double mx = -INFINITY;
        for (int64_t j = 0; j < jend; j++) {
            double acc = 0.0;
            for (int c = 0; c < d; c++)
                acc += Q[i * stride + c] * K[j * stride + c];
            s[j] = sm_scale * acc;
            if (s[j] > mx)
                mx = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < jend; j++) {
            s[j] = exp(s[j] - mx);
            l += s[j];
        }
        for (int c = 0; c < d; c++) {
            double o = 0.0;
            for (int64_t j = 0; j < jend; j++)
                o += s[j] * V[j * stride + c];
            out[i * stride + c] = o / l;
        }
        free(s);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
