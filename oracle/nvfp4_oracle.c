/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 block-scaled MoE path.
 *
 * TEST INFRASTRUCTURE. Only tests/, the smoke check and the benchmark's CPU
 * baseline leg may load this library. The product path never calls it and it
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources. The pages describe the workload, not the numerics:
 *   - "Peering into the CUTLASS Kernel Cache" (Knowledge Required, last item):
 *     NVFP4 packs two 4-bit values into each byte; the model is a
 *     Mixture-of-Experts whose grouped GEMM multiplies each expert's weight
 *     matrix by the subset of tokens routed to it.
 *   - "Peering into the CUTLASS SharedStorage" (Input Knowledge Required, item 3):
 *     FP4 values packed two per byte with one FP8 scale factor per block of 16
 *     elements; (item 5) the grouped GEMM batches one small GEMM per expert.
 *   - "Peering into the CUTLASS Kernel" (Input Knowledge Required, item 5): the
 *     FINALIZE epilogue performs the final MoE output write.
 * The problem statement fixes the rest: E2M1 elements, E4M3 block scales, an
 * FP32 per-tensor global scale, SwiGLU on gate/up and a top-k weighted combine.
 * Every step the pages leave open is taken in its plainest reading; the list of
 * readings is kept with the design notes (global scale = amax / (6 * 448)
 * stored as the dequantisation multiplier, FP32 round-to-nearest-even for the
 * scale and element arithmetic, satfinite conversions, sign kept on zero, even
 * element in the low nibble, gate rows first then up rows, stable (t, j)
 * expert order).
 *
 * Precision: codecs are written from the format definitions and evaluated
 * exactly in double; the quantiser performs the FP32 steps it is defined by
 * (build with -ffp-contract=off so no FMA contraction changes them); GEMM dot
 * products, SiLU and the combine accumulate in FP64; BF16 results are rounded
 * once, from FP64, to nearest-even.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* BF16                                                                      */
/* ------------------------------------------------------------------------ */

float oracle_bf16_to_float(uint16_t b) {
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* Round a double to the nearest BF16 (8 significant bits), ties to even,
 * in one step (no intermediate FP32 rounding). */
uint16_t oracle_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                /* a in [2^(e-1), 2^e) */
    int ulp_exp = e - 8;         /* 8 significant bits */
    if (ulp_exp < -133) ulp_exp = -133;  /* BF16 subnormal spacing 2^-133 */
    double r = ldexp(nearbyint(ldexp(a, -ulp_exp)), ulp_exp);  /* RNE */
    if (r > 3.3895313892515355e38) return sign | 0x7F80;        /* above max finite BF16 */
    float fr = (float)r;         /* exact: r has at most 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &fr, 4);
    return sign | (uint16_t)(bits >> 16);
}

void oracle_bf16_from_double_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = oracle_bf16_from_double(v[i]);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.        */
/* ------------------------------------------------------------------------ */

double oracle_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Round-to-nearest-even onto the E2M1 grid with saturation to +-6; the sign
 * of the input is kept, so a negative value that rounds to zero gives 0x8. */
uint8_t oracle_e2m1_encode(float y) {
    uint8_t sign = signbit(y) ? 0x8 : 0x0;
    double a = fabs((double)y);
    uint8_t c = 7; /* saturate unless a grid interval below claims it */
    for (uint8_t i = 0; i < 7; i++) {
        double lo = oracle_e2m1_decode(i), hi = oracle_e2m1_decode((uint8_t)(i + 1));
        double mid = 0.5 * (lo + hi);
        if (a < mid) { c = i; break; }
        if (a == mid) { c = (i % 2 == 0) ? i : (uint8_t)(i + 1); break; }  /* even mantissa */
    }
    return sign | c;
}

/* ------------------------------------------------------------------------ */
/* E4M3 (FP8): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits,       */
/* subnormals m * 2^-9, max finite 448, S.1111.111 is NaN, no infinities.   */
/* ------------------------------------------------------------------------ */

double oracle_e4m3_decode(uint8_t b) {
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating to +-448 (satfinite). */
uint8_t oracle_e4m3_encode(float s) {
    uint8_t sign = signbit(s) ? 0x80 : 0x00;
    double a = fabs((double)s);
    uint8_t c = 126; /* 0x7E = 448, the largest finite magnitude */
    for (uint8_t i = 0; i < 126; i++) {
        double lo = oracle_e4m3_decode(i), hi = oracle_e4m3_decode((uint8_t)(i + 1));
        double mid = 0.5 * (lo + hi);
        if (a < mid) { c = i; break; }
        if (a == mid) { c = (i % 2 == 0) ? i : (uint8_t)(i + 1); break; }
    }
    return sign | c;
}

/* ------------------------------------------------------------------------ */
/* Quantisation of one tensor X [rows, K] (K % 16 == 0).                    */
/*   amax_t = max|x|; g_enc = 2688 / amax_t, g_dec = amax_t / 2688           */
/*   (2688 = 6 * 448, the E2M1 maximum times the E4M3 maximum; all-zero      */
/*   tensor: both 1). A caller-given global scale is g_dec, g_enc = 1/g_dec. */
/*   Per 16-element block: s = (amax_b / 6) * g_enc -> S = E4M3(s);         */
/*   S == 0 -> all codes +0; else f = g_enc / float(S), code = E2M1(x * f).  */
/*   Output: q [rows, K/2] (element 2i low nibble), sf [rows, K/16] row-major,*/
/*   *gdec_out = g_dec.                                                      */
/* ------------------------------------------------------------------------ */

float oracle_amax(const uint16_t* x, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(oracle_bf16_to_float(x[i]));
        if (a > amax) amax = a;
    }
    return amax;
}

void oracle_global_scales(float amax, const float* gdec_in, float* g_enc, float* g_dec) {
    volatile float num = 2688.0f;
    if (gdec_in) {
        *g_dec = *gdec_in;
        *g_enc = 1.0f / *g_dec;
    } else if (amax == 0.0f) {
        *g_enc = 1.0f;
        *g_dec = 1.0f;
    } else {
        *g_enc = num / amax;
        *g_dec = amax / num;
    }
}

static void quantize_block(const uint16_t* xb, float g_enc, uint8_t* qb, uint8_t* sfb) {
    float amax_b = 0.0f;
    for (int i = 0; i < 16; i++) {
        float a = fabsf(oracle_bf16_to_float(xb[i]));
        if (a > amax_b) amax_b = a;
    }
    volatile float t = amax_b / 6.0f;      /* FP32 RN, then */
    float s = t * g_enc;                    /* FP32 RN, separately rounded */
    uint8_t S = oracle_e4m3_encode(s);
    *sfb = S;
    float sfv = (float)oracle_e4m3_decode(S);
    uint8_t codes[16];
    if (sfv == 0.0f) {
        for (int i = 0; i < 16; i++) codes[i] = 0;
    } else {
        volatile float f = g_enc / sfv;     /* one FP32 RN division per block */
        for (int i = 0; i < 16; i++) {
            float y = oracle_bf16_to_float(xb[i]) * f;
            codes[i] = oracle_e2m1_encode(y);
        }
    }
    for (int i = 0; i < 8; i++) qb[i] = (uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4));
}

void oracle_quantize(const uint16_t* x, int64_t rows, int64_t K, const float* gdec_in,
                     uint8_t* q, uint8_t* sf, float* gdec_out) {
    float amax = gdec_in ? 0.0f : oracle_amax(x, rows * K);
    float g_enc, g_dec;
    oracle_global_scales(amax, gdec_in, &g_enc, &g_dec);
    int64_t nblk = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nblk; b++) {
            quantize_block(x + r * K + b * 16, g_enc, q + r * (K / 2) + b * 8, sf + r * nblk + b);
        }
    }
    if (gdec_out) *gdec_out = g_dec;
}

/* Quantisation with the tensor amax supplied by the caller: the same steps as
 * oracle_quantize, for a tensor whose rows are spread over several places (one
 * global scale for the whole tensor: its amax is the max over all parts). */
void oracle_quantize_amax(const uint16_t* x, int64_t rows, int64_t K, float amax,
                          uint8_t* q, uint8_t* sf, float* gdec_out) {
    float g_enc, g_dec;
    oracle_global_scales(amax, NULL, &g_enc, &g_dec);
    int64_t nblk = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t b = 0; b < nblk; b++) {
            quantize_block(x + r * K + b * 16, g_enc, q + r * (K / 2) + b * 8, sf + r * nblk + b);
        }
    }
    if (gdec_out) *gdec_out = g_dec;
}

/* Decoded-value tables, filled from the decode functions above. */
static double E2M1_VAL[16];
static double E4M3_VAL[256];
static int tables_ready = 0;

static void init_tables(void) {
    if (tables_ready) return;
    for (int c = 0; c < 16; c++) E2M1_VAL[c] = oracle_e2m1_decode((uint8_t)c);
    for (int b = 0; b < 256; b++) E4M3_VAL[b] = oracle_e4m3_decode((uint8_t)b);
    tables_ready = 1;
}

/* Dequantised element value without the global scale: E2M1(code) * E4M3(S). */
static double dq_elem(const uint8_t* q_row, const uint8_t* sf_row, int64_t k) {
    uint8_t byte = q_row[k >> 1];
    uint8_t code = (k & 1) ? (byte >> 4) : (byte & 15);
    return E2M1_VAL[code] * E4M3_VAL[sf_row[k >> 4]];
}

static void dq_row(const uint8_t* q_row, const uint8_t* sf_row, int64_t K, double* out) {
    for (int64_t k = 0; k < K; k++) out[k] = dq_elem(q_row, sf_row, k);
}

void oracle_dequantize(const uint8_t* q, const uint8_t* sf, float g_dec, int64_t rows, int64_t K,
                       double* out) {
    init_tables();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K; k++)
            out[r * K + k] = dq_elem(q + r * (K / 2), sf + r * (K / 16), k) * (double)g_dec;
}

/* ------------------------------------------------------------------------ */
/* Routing: explicit counting, stable in (t ascending, j ascending).        */
/* ------------------------------------------------------------------------ */

int oracle_permute(const int32_t* ids, int32_t T, int32_t k, int32_t E,
                   int32_t* offsets, int32_t* perm_src, int32_t* inv_perm) {
    int32_t* fill = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
    if (!fill) return -1;
    for (int32_t e = 0; e <= E; e++) offsets[e] = 0;
    for (int64_t i = 0; i < (int64_t)T * k; i++) {
        int32_t e = ids[i];
        if (e < 0 || e >= E) { free(fill); return -2; }
        offsets[e + 1] += 1;
    }
    for (int32_t e = 0; e < E; e++) offsets[e + 1] += offsets[e];
    for (int32_t e = 0; e < E; e++) fill[e] = offsets[e];
    for (int32_t t = 0; t < T; t++) {
        for (int32_t j = 0; j < k; j++) {
            int32_t e = ids[(int64_t)t * k + j];
            int32_t p = fill[e]++;
            perm_src[p] = t;
            inv_perm[(int64_t)t * k + j] = p;
        }
    }
    free(fill);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Router: top-k experts of each token by logit, then the softmax of the    */
/* chosen logits. The pages do not describe the router; the MoE grouped     */
/* GEMM only needs "the subset of tokens routed to" each expert ("Peering   */
/* into the CUTLASS Kernel Cache", Knowledge Required). Reading taken: the  */
/* k largest logits by value, the lower expert index first among equal      */
/* values (+0 and -0 are equal), listed in that order; weights = softmax    */
/* over the whole row restricted to the chosen k and renormalised, which is */
/* the softmax of the k chosen logits alone:                                */
/*   w[t, j] = exp(z[ids[t, j]] - m) / sum_i exp(z[ids[t, i]] - m),         */
/*   m = z[ids[t, 0]], the sum over i ascending, all in FP64, rounded once  */
/*   to FP32. A token whose largest chosen logit is -inf gets 1/k each.     */
/* Logits are finite or -inf (no NaN, no +inf); 1 <= k <= E.                */
/* ------------------------------------------------------------------------ */

void oracle_route_topk(const float* z, int32_t T, int32_t E, int32_t k, int32_t* ids, float* w) {
    unsigned char* taken = (unsigned char*)malloc((size_t)E);
    double* ex = (double*)malloc(sizeof(double) * (size_t)k);
    for (int32_t t = 0; t < T; t++) {
        const float* zt = z + (int64_t)t * E;
        int32_t* it = ids + (int64_t)t * k;
        memset(taken, 0, (size_t)E);
        /* explicit selection: k passes, each picking the largest untaken logit */
        for (int32_t j = 0; j < k; j++) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || zt[e] > zt[best]) best = e;   /* strict: an equal later value never wins */
            }
            taken[best] = 1;
            it[j] = best;
        }
        const double m = (double)zt[it[0]];
        if (isinf(m) && m < 0) {
            for (int32_t j = 0; j < k; j++) w[(int64_t)t * k + j] = (float)(1.0 / (double)k);
            continue;
        }
        double sum = 0.0;
        for (int32_t j = 0; j < k; j++) {
            ex[j] = exp((double)zt[it[j]] - m);
            sum += ex[j];
        }
        for (int32_t j = 0; j < k; j++) w[(int64_t)t * k + j] = (float)(ex[j] / sum);
    }
    free(ex);
    free(taken);
}

/* Row gather: dst row p is a byte copy of src row idx[p]. */
void oracle_gather_rows(const uint8_t* src, int64_t row_bytes, const int32_t* idx, int64_t n,
                        uint8_t* dst) {
    for (int64_t p = 0; p < n; p++) memcpy(dst + p * row_bytes, src + (int64_t)idx[p] * row_bytes, (size_t)row_bytes);
}

/* ------------------------------------------------------------------------ */
/* Grouped GEMM. Expert e owns activation rows [off[e], off[e+1]).           */
/*   acc[m, n] = sum_k A(m,k) * W_e(n,k)   (block-scaled values, FP64)       */
/*   alpha = g_dec_A * g_dec_W[e]                                            */
/*   epi 0 (NONE):   out[m, n] = alpha * acc[m, n],               n < N      */
/*   epi 1 (SWIGLU): out[m, n] = silu(alpha * acc[m, n]) * alpha * acc[m, N/2 + n],  */
/*                   n < N/2, silu(v) = v / (1 + exp(-v)); gate rows first.  */
/* Weights: w_q [E, N, K/2], w_sf [E, N, K/16] row-major, w_g [E].           */
/* ------------------------------------------------------------------------ */

static double silu(double v) { return v / (1.0 + exp(-v)); }

static double dot(const double* a, const double* b, int64_t K) {
    double acc = 0.0;
    for (int64_t k = 0; k < K; k++) acc += a[k] * b[k];
    return acc;
}

/* Full output for every routed row: out [off[E], Nout] FP64. */
void oracle_grouped_gemm(const uint8_t* a_q, const uint8_t* a_sf, float a_g,
                         const uint8_t* w_q, const uint8_t* w_sf, const float* w_g,
                         const int32_t* off, int32_t E, int64_t N, int64_t K, int32_t epi,
                         double* out) {
    init_tables();
    int64_t Nout = epi == 1 ? N / 2 : N;
    for (int32_t e = 0; e < E; e++) {
        int64_t m0 = off[e], M = off[e + 1] - off[e];
        if (M <= 0) continue;
        double alpha = (double)a_g * (double)w_g[e];
        double* A = (double*)malloc((size_t)(M * K) * sizeof(double));
        for (int64_t m = 0; m < M; m++)
            dq_row(a_q + (m0 + m) * (K / 2), a_sf + (m0 + m) * (K / 16), K, A + m * K);
        const uint8_t* wq = w_q + (int64_t)e * N * (K / 2);
        const uint8_t* wsf = w_sf + (int64_t)e * N * (K / 16);
#pragma omp parallel
        {
            double* wg = (double*)malloc((size_t)K * sizeof(double));
            double* wu = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(static)
            for (int64_t n = 0; n < Nout; n++) {
                dq_row(wq + n * (K / 2), wsf + n * (K / 16), K, wg);
                if (epi == 1) dq_row(wq + (N / 2 + n) * (K / 2), wsf + (N / 2 + n) * (K / 16), K, wu);
                for (int64_t m = 0; m < M; m++) {
                    double v = alpha * dot(A + m * K, wg, K);
                    if (epi == 1) v = silu(v) * (alpha * dot(A + m * K, wu, K));
                    out[(m0 + m) * Nout + n] = v;
                }
            }
            free(wg);
            free(wu);
        }
        free(A);
    }
}

static int32_t expert_of_row(const int32_t* off, int32_t E, int64_t row) {
    for (int32_t e = 0; e < E; e++)
        if (row >= off[e] && row < off[e + 1]) return e;
    return -1;
}

static double dot_row(const uint8_t* aq, const uint8_t* asf, const uint8_t* wq, const uint8_t* wsf,
                      int64_t K) {
    double acc = 0.0;
    for (int64_t k = 0; k < K; k++) acc += dq_elem(aq, asf, k) * dq_elem(wq, wsf, k);
    return acc;
}

/* Selected entries only: out[i] = result at (rows[i], cols[i]). */
void oracle_grouped_gemm_at(const uint8_t* a_q, const uint8_t* a_sf, float a_g,
                            const uint8_t* w_q, const uint8_t* w_sf, const float* w_g,
                            const int32_t* off, int32_t E, int64_t N, int64_t K, int32_t epi,
                            const int64_t* rows, const int64_t* cols, int64_t n_pts, double* out) {
    init_tables();
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n_pts; i++) {
        int64_t m = rows[i], n = cols[i];
        int32_t e = expert_of_row(off, E, m);
        if (e < 0) { out[i] = NAN; continue; }
        double alpha = (double)a_g * (double)w_g[e];
        const uint8_t* aq = a_q + m * (K / 2);
        const uint8_t* asf = a_sf + m * (K / 16);
        const uint8_t* wq = w_q + (int64_t)e * N * (K / 2);
        const uint8_t* wsf = w_sf + (int64_t)e * N * (K / 16);
        double v = alpha * dot_row(aq, asf, wq + n * (K / 2), wsf + n * (K / 16), K);
        if (epi == 1) {
            double u = alpha * dot_row(aq, asf, wq + (N / 2 + n) * (K / 2), wsf + (N / 2 + n) * (K / 16), K);
            v = silu(v) * u;
        }
        out[i] = v;
    }
}

/* ------------------------------------------------------------------------ */
/* FP32 error bound of a GEMM output computed the way a tensor-core path    */
/* computes it (test infrastructure: it decides which one-ulp BF16          */
/* disagreements are rounding ties, not what the result is).               */
/* Model: a 16-element block's partial P_b = sum of its 16 products of      */
/* decoded values is exact in FP32 (E2M1 x E2M1 products are multiples of  */
/* 1/4 below 37, so their sum needs at most 11 bits, times an E4M3 x E4M3   */
/* scale product of at most 8 significant bits); the K/16 partials are      */
/* accumulated in FP32; alpha = FP32(g_A * g_W) and alpha * acc are FP32    */
/* products; SwiGLU uses single-precision fast exp and division. First-     */
/* order bounds, u = 2^-24, gamma_n = n u / (1 - n u):                       */
/*   NONE:   |y' - y| <= |alpha| gamma_{K/16} sum_b |P_b| (1 + 2u)          */
/*                       + 2.01 u |alpha acc|                                */
/*   SWIGLU: with dg, du the NONE bounds of gate and up,                    */
/*           |h' - h| <= 1.1 dg (|up| + du) + |silu(gate)| du               */
/*                       + (8 + 2 |gate|) 2^-23 |h|                          */
/*   (1.1 bounds |silu'|; the last term covers the fast exp and division.)  */
/* ------------------------------------------------------------------------ */

static double block_dot(const double* a, const double* w, int64_t K, double* sabs) {
    double acc = 0.0, t = 0.0;
    for (int64_t b = 0; b < K / 16; b++) {
        double p = 0.0;
        for (int i = 0; i < 16; i++) p += a[b * 16 + i] * w[b * 16 + i];
        acc += p;
        t += fabs(p);
    }
    *sabs = t;
    return acc;
}

static double bound_plain(double alpha, double acc, double sabs, int64_t K) {
    const double u = 5.9604644775390625e-08, nu = (double)(K / 16) * u;
    return fabs(alpha) * (nu / (1.0 - nu)) * sabs * (1.0 + 2.0 * u) + 2.01 * u * fabs(alpha * acc);
}

static double bound_swiglu(double alpha, double accg, double sg, double accu, double su, int64_t K) {
    const double g = alpha * accg, up = alpha * accu;
    const double dg = bound_plain(alpha, accg, sg, K), du = bound_plain(alpha, accu, su, K);
    const double h = silu(g) * up;
    return 1.1 * dg * (fabs(up) + du) + fabs(silu(g)) * du + (8.0 + 2.0 * fabs(g)) * 1.1920928955078125e-07 * fabs(h);
}

/* Bound of every output of oracle_grouped_gemm (same arguments), bound [off[E], Nout]. */
void oracle_grouped_gemm_bound(const uint8_t* a_q, const uint8_t* a_sf, float a_g,
                               const uint8_t* w_q, const uint8_t* w_sf, const float* w_g,
                               const int32_t* off, int32_t E, int64_t N, int64_t K, int32_t epi,
                               double* bound) {
    init_tables();
    int64_t Nout = epi == 1 ? N / 2 : N;
    for (int32_t e = 0; e < E; e++) {
        int64_t m0 = off[e], M = off[e + 1] - off[e];
        if (M <= 0) continue;
        double alpha = (double)a_g * (double)w_g[e];
        double* A = (double*)malloc((size_t)(M * K) * sizeof(double));
        for (int64_t m = 0; m < M; m++)
            dq_row(a_q + (m0 + m) * (K / 2), a_sf + (m0 + m) * (K / 16), K, A + m * K);
        const uint8_t* wq = w_q + (int64_t)e * N * (K / 2);
        const uint8_t* wsf = w_sf + (int64_t)e * N * (K / 16);
#pragma omp parallel
        {
            double* wg = (double*)malloc((size_t)K * sizeof(double));
            double* wu = (double*)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(static)
            for (int64_t n = 0; n < Nout; n++) {
                dq_row(wq + n * (K / 2), wsf + n * (K / 16), K, wg);
                if (epi == 1) dq_row(wq + (N / 2 + n) * (K / 2), wsf + (N / 2 + n) * (K / 16), K, wu);
                for (int64_t m = 0; m < M; m++) {
                    double sg, su;
                    const double ag = block_dot(A + m * K, wg, K, &sg);
                    double b;
                    if (epi == 1) {
                        const double au = block_dot(A + m * K, wu, K, &su);
                        b = bound_swiglu(alpha, ag, sg, au, su, K);
                    } else {
                        b = bound_plain(alpha, ag, sg, K);
                    }
                    bound[(m0 + m) * Nout + n] = b;
                }
            }
            free(wg);
            free(wu);
        }
        free(A);
    }
}

/* Bound at the selected (row, col) points only (same arguments as oracle_grouped_gemm_at). */
static double block_dot_row(const uint8_t* aq, const uint8_t* asf, const uint8_t* wq, const uint8_t* wsf,
                            int64_t K, double* sabs) {
    double acc = 0.0, t = 0.0;
    for (int64_t b = 0; b < K / 16; b++) {
        double p = 0.0;
        for (int64_t k = b * 16; k < b * 16 + 16; k++) p += dq_elem(aq, asf, k) * dq_elem(wq, wsf, k);
        acc += p;
        t += fabs(p);
    }
    *sabs = t;
    return acc;
}

void oracle_grouped_gemm_bound_at(const uint8_t* a_q, const uint8_t* a_sf, float a_g,
                                  const uint8_t* w_q, const uint8_t* w_sf, const float* w_g,
                                  const int32_t* off, int32_t E, int64_t N, int64_t K, int32_t epi,
                                  const int64_t* rows, const int64_t* cols, int64_t n_pts, double* bound) {
    init_tables();
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n_pts; i++) {
        int64_t m = rows[i], n = cols[i];
        int32_t e = expert_of_row(off, E, m);
        if (e < 0) { bound[i] = NAN; continue; }
        double alpha = (double)a_g * (double)w_g[e];
        const uint8_t* aq = a_q + m * (K / 2);
        const uint8_t* asf = a_sf + m * (K / 16);
        const uint8_t* wq = w_q + (int64_t)e * N * (K / 2);
        const uint8_t* wsf = w_sf + (int64_t)e * N * (K / 16);
        double sg, su;
        const double ag = block_dot_row(aq, asf, wq + n * (K / 2), wsf + n * (K / 16), K, &sg);
        if (epi == 1) {
            const double au = block_dot_row(aq, asf, wq + (N / 2 + n) * (K / 2), wsf + (N / 2 + n) * (K / 16), K, &su);
            bound[i] = bound_swiglu(alpha, ag, sg, au, su, K);
        } else {
            bound[i] = bound_plain(alpha, ag, sg, K);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Top-k weighted combine: out[t, h] = sum_j w[t, j] * y[inv_perm[t*k+j], h] */
/* accumulated in FP64 over j ascending.                                    */
/* ------------------------------------------------------------------------ */

void oracle_combine(const uint16_t* y, const int32_t* inv_perm, const float* w,
                    int32_t T, int32_t k, int64_t H, double* out) {
#pragma omp parallel for schedule(static)
    for (int32_t t = 0; t < T; t++) {
        for (int64_t h = 0; h < H; h++) {
            double acc = 0.0;
            for (int32_t j = 0; j < k; j++) {
                int64_t p = inv_perm[(int64_t)t * k + j];
                if (p < 0) continue;   /* a pair without an expert row (the permute's -1) adds nothing */
                acc += (double)w[(int64_t)t * k + j] * (double)oracle_bf16_to_float(y[p * H + h]);
            }
            out[(int64_t)t * H + h] = acc;
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
