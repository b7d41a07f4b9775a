/*
 * moe_oracle.c -- plain, slow CPU oracle for the forward pass of a MoE layer with
 * zero-computation experts, and for its expert-bias update.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg load this library. The CUDA path never links, loads or calls it, and it shares no
 * source with the CUDA path.
 *
 * What it follows (all from the LongCat-Flash llm-wiki entity page):
 *   - section 2.1 "Zero-Computation Experts", MoE equation: MoE(x_t) = sum_{i=1}^{N+Z} g_i E_i(x_t),
 *     experts 0..N-1 are FFN experts, N..N+Z-1 are zero-computation experts with E_i(x_t) = x_t;
 *   - section 2.1, dynamic computation-budget control: the router picks K experts per token
 *     (zero experts included) steered by per-expert biases b_i, updated by
 *     delta_b_i = mu * (K_e/K * 1/N - T_i / (K * T_all));
 *   - section 2.3.2, expert-initialisation variance compensation: the gate is a softmax;
 *   - section 1, core-parameter table: FFN-expert width, expert counts, K = 12 including zero
 *     experts.
 * Readings where the page is silent (each is listed with its reason in the design notes):
 *   softmax over all N+Z experts; bias added to the softmax scores for selection only; gates are
 *   the unbiased scores renormalised over the K chosen; ties go to the lower index; SwiGLU
 *   experts with three d x I matrices; bf16 rounding at H, Y and the output; fp32 for logits,
 *   scores, gates and the bias arithmetic; the bias rule applied to all N+Z experts.
 *
 * Floating point: accumulations are in double unless a step is specified in fp32. Compile
 * with -ffp-contract=off and without fast-math: every fp32 step below is one IEEE
 * round-to-nearest operation, fmaf only where written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ABI_VERSION 1

int oracle_abi_version(void) { return ORACLE_ABI_VERSION; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------------ */
/* bf16 helpers: a bf16 value is the upper 16 bits of an IEEE binary32.                        */
/* ------------------------------------------------------------------------------------------ */

static double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double directly to the nearest bf16 value, ties to even (one rounding). */
uint16_t oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    /* halfway between the largest finite bf16 (0x1.fep127) and 2^128 rounds to infinity */
    if (a >= 0x1.ffp127) return (uint16_t)(sign | 0x7F80);
    int e;
    (void)frexp(a, &e);              /* a = m * 2^e, m in [0.5, 1) */
    int shift = e - 8;               /* 8 significant bits */
    if (shift < -133) shift = -133;  /* subnormal spacing of bf16 */
    double q = rint(ldexp(a, -shift));   /* default rounding mode: nearest, ties to even */
    float r = (float)ldexp(q, shift);    /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &r, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

double oracle_bf16_to_double(uint16_t h) { return bf16_to_double(h); }

/* ------------------------------------------------------------------------------------------ */
/* Step 1: router logits  z[t,i] = sum_j x[t,j] * Wr[i,j]   (double, then one rounding to fp32) */
/* ------------------------------------------------------------------------------------------ */

void oracle_router_logits(const uint16_t* x, const uint16_t* wr, int64_t T, int64_t d, int64_t E,
                          float* z) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < E; ++i) {
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j)
                acc += bf16_to_double(x[t * d + j]) * bf16_to_double(wr[i * d + j]);
            z[t * E + i] = (float)acc;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Project-specified exp and sum for the softmax (so that a GPU kernel written separately from */
/* the same specification reproduces the scores bit for bit).                                  */
/*                                                                                             */
/* EXP(u): Cody-Waite argument reduction (Cody & Waite, "Software Manual for the Elementary    */
/* Functions", 1980) u = n ln2 + r with n = rint(u log2 e) and ln 2 split in a 16-bit head and */
/* a tail, then the degree-7 Taylor polynomial of e^r (coefficients 1/k!) by Horner's rule     */
/* with fused multiply-adds, scaled by 2^n. Inputs below -86 give 0, so every non-zero result  */
/* is a normal number and the final scaling is exact.                                          */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    float log2e, ln2_hi, ln2_lo;
    float c[8];
} exp_consts;

static exp_consts make_exp_consts(void) {
    exp_consts k;
    const double ln2 = 0.693147180559945309417232121458176568;  /* ln 2 */
    k.log2e = (float)(1.0 / ln2);
    double hi = ldexp(rint(ldexp(ln2, 16)), -16);   /* ln 2 rounded to 16 fraction bits */
    k.ln2_hi = (float)hi;                            /* exact */
    k.ln2_lo = (float)(ln2 - hi);
    double f = 1.0;
    for (int i = 0; i < 8; ++i) {                   /* 1/k! */
        if (i > 0) f *= (double)i;
        k.c[i] = (float)(1.0 / f);
    }
    return k;
}

static exp_consts K_EXP;
__attribute__((constructor)) static void init_exp_consts(void) { K_EXP = make_exp_consts(); }

float oracle_exp_spec(float u) {
    const exp_consts K = K_EXP;
    if (isnan(u)) return u;
    if (u < -86.0f) return 0.0f;
    if (u > 88.0f) return INFINITY;
    float n = rintf(u * K.log2e);
    float r = fmaf(-n, K.ln2_hi, u);
    r = fmaf(-n, K.ln2_lo, r);
    float p = K.c[7];
    for (int i = 6; i >= 0; --i) p = fmaf(p, r, K.c[i]);
    int ni = (int)n;
    uint32_t bits = (uint32_t)(ni + 127) << 23;     /* 2^n, a normal number for n in [-124, 127] */
    float scale;
    memcpy(&scale, &bits, sizeof scale);
    return p * scale;
}

/* SUM over E values: 32 partial sums, partial l adds v[l], v[l+32], v[l+64], ... in order
 * (starting from +0), then five pairwise rounds where partial l becomes
 * partial[l] + partial[l ^ off] for off = 16, 8, 4, 2, 1. Every partial ends equal; the result
 * is partial 0. */
float oracle_sum_spec(const float* v, int64_t E) {
    float p[32];
    for (int l = 0; l < 32; ++l) {
        float acc = 0.0f;
        for (int64_t j = l; j < E; j += 32) acc = acc + v[j];
        p[l] = acc;
    }
    for (int off = 16; off >= 1; off >>= 1) {
        float q[32];
        for (int l = 0; l < 32; ++l) q[l] = p[l] + p[l ^ off];
        memcpy(p, q, sizeof p);
    }
    return p[0];
}

/* ------------------------------------------------------------------------------------------ */
/* Steps 2-5: softmax scores, biased top-K selection, gates, expert counts.                    */
/* ------------------------------------------------------------------------------------------ */

/* For every token: s = softmax(z) over all E experts (EXP/SUM above, IEEE divide);
 * key_i = s_i + b_i; the K largest keys in descending order, equal keys to the lower index;
 * g_r = s_sel[r] / Q with Q = s_sel[0] + ... + s_sel[K-1] summed in rank order.
 * counts[i] (length E) is ADDED TO with the number of (token, rank) picks of expert i.
 * scores (optional, [T,E]) receives s. Returns 0, or the number of tokens whose keys held a
 * NaN (their picks are then the K lowest indices and their gates NaN). */
int64_t oracle_route(const float* z, const float* bias, int64_t T, int64_t E, int64_t K,
                     int32_t* idx, float* gate, int32_t* counts, float* scores) {
    int64_t bad = 0;
    #pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t t = 0; t < T; ++t) {
        const float* zt = z + t * E;
        float* e = (float*)malloc((size_t)E * sizeof(float));
        float* s = (float*)malloc((size_t)E * sizeof(float));
        float* key = (float*)malloc((size_t)E * sizeof(float));
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        /* max over the logits; a NaN logit is skipped here and turns every key into NaN below */
        float m = -INFINITY;
        for (int64_t i = 0; i < E; ++i)
            if (zt[i] > m) m = zt[i];
        for (int64_t i = 0; i < E; ++i) e[i] = oracle_exp_spec(zt[i] - m);
        float S = oracle_sum_spec(e, E);
        int nan_key = 0;
        for (int64_t i = 0; i < E; ++i) {
            s[i] = e[i] / S;
            key[i] = s[i] + bias[i];
            if (isnan(key[i])) nan_key = 1;
        }
        if (scores) memcpy(scores + t * E, s, (size_t)E * sizeof(float));
        if (nan_key) {
            bad += 1;
            for (int64_t r = 0; r < K; ++r) { idx[t * K + r] = (int32_t)r; gate[t * K + r] = NAN; }
        } else {
            float Q = 0.0f;
            for (int64_t r = 0; r < K; ++r) {
                int64_t best = -1;
                for (int64_t i = 0; i < E; ++i) {
                    if (taken[i]) continue;
                    /* strictly greater: scanning upwards, an equal key keeps the lower index */
                    if (best < 0 || key[i] > key[best]) best = i;
                }
                taken[best] = 1;
                idx[t * K + r] = (int32_t)best;
                Q = Q + s[best];
            }
            for (int64_t r = 0; r < K; ++r) gate[t * K + r] = s[idx[t * K + r]] / Q;
        }
        free(e); free(s); free(key); free(taken);
    }
    if (counts)
        for (int64_t t = 0; t < T; ++t)
            for (int64_t r = 0; r < K; ++r) counts[idx[t * K + r]] += 1;
    return bad;
}

/* ------------------------------------------------------------------------------------------ */
/* Step 6: grouping of the (token, rank) pairs routed to FFN experts.                          */
/* Rows are ordered by expert, and by token inside an expert (each token picks an expert at    */
/* most once). offsets[e] is the first row of expert e, offsets[N] the number of rows M.       */
/* pair_row[t,r] is the row of pick (t,r), or -1 if that pick is a zero-computation expert.    */
/* Returns M.                                                                                  */
/* ------------------------------------------------------------------------------------------ */

int64_t oracle_permute(const int32_t* idx, int64_t T, int64_t K, int64_t N,
                       int32_t* offsets, int32_t* row_token, int32_t* pair_row) {
    for (int64_t p = 0; p < T * K; ++p) pair_row[p] = -1;
    int64_t pos = 0;
    for (int64_t e = 0; e < N; ++e) {
        offsets[e] = (int32_t)pos;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t r = 0; r < K; ++r)
                if (idx[t * K + r] == e) {
                    row_token[pos] = (int32_t)t;
                    pair_row[t * K + r] = (int32_t)pos;
                    ++pos;
                }
    }
    offsets[N] = (int32_t)pos;
    return pos;
}

/* ------------------------------------------------------------------------------------------ */
/* Step 7: FFN experts (SwiGLU).  For a row x routed to expert e:                              */
/*   G_j = sum_k x_k Wg[e][j][k],  U_j = sum_k x_k Wu[e][j][k]      (j < I, double)            */
/*   H_j = bf16( G_j * sigmoid(G_j) * U_j )                                                    */
/*   Y_i = bf16( sum_j H_j Wd[e][i][j] )                           (i < d, double)             */
/* with W13[e] = [Wg[e]; Wu[e]] of shape [2I, d] and W2[e] = Wd[e] of shape [d, I].            */
/* row_expert[r] selects the expert of row r; w13/w2 may point at a single expert with all     */
/* row_expert 0.                                                                               */
/* ------------------------------------------------------------------------------------------ */

/* Down projection of one row: Y_i = bf16( sum_j H_j Wd[i][j] ), double accumulation. */
static void down_row(const double* hd, const uint16_t* wd, int64_t d, int64_t I, uint16_t* yrow) {
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < I; ++j) acc += hd[j] * bf16_to_double(wd[i * I + j]);
        yrow[i] = oracle_double_to_bf16(acc);
    }
}

void oracle_expert_rows(const uint16_t* xrows, const int32_t* row_expert, int64_t M, int64_t d,
                        int64_t I, const uint16_t* w13, const uint16_t* w2, uint16_t* h,
                        uint16_t* y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        const int64_t e = row_expert[r];
        const uint16_t* xr = xrows + r * d;
        const uint16_t* wg = w13 + e * 2 * I * d;
        const uint16_t* wu = wg + I * d;
        const uint16_t* wd = w2 + e * d * I;
        double* xd = (double*)malloc((size_t)d * sizeof(double));
        double* hd = (double*)malloc((size_t)I * sizeof(double));
        for (int64_t k = 0; k < d; ++k) xd[k] = bf16_to_double(xr[k]);
        for (int64_t j = 0; j < I; ++j) {
            double G = 0.0, U = 0.0;
            for (int64_t k = 0; k < d; ++k) {
                G += xd[k] * bf16_to_double(wg[j * d + k]);
                U += xd[k] * bf16_to_double(wu[j * d + k]);
            }
            double act = G / (1.0 + exp(-G));   /* G * sigmoid(G) */
            uint16_t hb = oracle_double_to_bf16(act * U);
            if (h) h[r * I + j] = hb;
            hd[j] = bf16_to_double(hb);
        }
        down_row(hd, wd, d, I, y + r * d);
        free(xd); free(hd);
    }
}

/* The down projection alone, from given bf16 rows H [M, I]: Y = bf16(H Wd[e]^T). */
void oracle_expert_down(const uint16_t* h, const int32_t* row_expert, int64_t M, int64_t d,
                        int64_t I, const uint16_t* w2, uint16_t* y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        double* hd = (double*)malloc((size_t)I * sizeof(double));
        for (int64_t j = 0; j < I; ++j) hd[j] = bf16_to_double(h[r * I + j]);
        down_row(hd, w2 + (int64_t)row_expert[r] * d * I, d, I, y + r * d);
        free(hd);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Step 8: combine. out_t = bf16( sum_r g_r * v_r ), v_r = Y[pair_row[t,r]] for an FFN pick    */
/* and v_r = x_t for a zero-computation pick (E_i(x) = x), summed in double in rank order.     */
/* out_acc (optional, [T, d]) receives the double sum before its rounding to bf16.             */
/* ------------------------------------------------------------------------------------------ */

void oracle_combine(const uint16_t* x, const uint16_t* y, const int32_t* idx, const float* gate,
                    const int32_t* pair_row, int64_t T, int64_t d, int64_t K, int64_t N,
                    uint16_t* out, double* out_acc) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t r = 0; r < K; ++r) {
                double g = (double)gate[t * K + r];
                double v = (idx[t * K + r] < N) ? bf16_to_double(y[(int64_t)pair_row[t * K + r] * d + c])
                                                : bf16_to_double(x[t * d + c]);
                acc += g * v;
            }
            out[t * d + c] = oracle_double_to_bf16(acc);
            if (out_acc) out_acc[t * d + c] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* The whole layer, straight from the MoE equation: each token's output is the gate-weighted   */
/* sum of its K chosen experts applied to it (no grouping step). logits/idx/gate are outputs;  */
/* counts (length E) is ADDED TO; out_acc (optional) receives the double sums before rounding. */
/* Returns the number of tokens with a NaN key.                                                */
/* ------------------------------------------------------------------------------------------ */

int64_t oracle_forward(const uint16_t* x, const uint16_t* wr, const float* bias,
                       const uint16_t* w13, const uint16_t* w2, int64_t T, int64_t d, int64_t N,
                       int64_t Z, int64_t K, int64_t I, uint16_t* out, float* logits, int32_t* idx,
                       float* gate, int32_t* counts, double* out_acc) {
    const int64_t E = N + Z;
    oracle_router_logits(x, wr, T, d, E, logits);
    int64_t bad = oracle_route(logits, bias, T, E, K, idx, gate, counts, NULL);
    for (int64_t t = 0; t < T; ++t) {
        double* acc = (double*)calloc((size_t)d, sizeof(double));
        uint16_t* yrow = (uint16_t*)malloc((size_t)d * sizeof(uint16_t));
        for (int64_t r = 0; r < K; ++r) {
            const int32_t e = idx[t * K + r];
            const double g = (double)gate[t * K + r];
            if (e < N) {
                oracle_expert_rows(x + t * d, &e, 1, d, I, w13, w2, NULL, yrow);
                for (int64_t c = 0; c < d; ++c) acc[c] += g * bf16_to_double(yrow[c]);
            } else {
                for (int64_t c = 0; c < d; ++c) acc[c] += g * bf16_to_double(x[t * d + c]);
            }
        }
        for (int64_t c = 0; c < d; ++c) {
            out[t * d + c] = oracle_double_to_bf16(acc[c]);
            if (out_acc) out_acc[t * d + c] = acc[c];
        }
        free(acc); free(yrow);
    }
    return bad;
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 experts. The LongCat-Flash llm-wiki entity page, section 5 (inference and deployment),   */
/* lists FP8/BF16 quantisation among the system-level optimisations and an FP8 deployment on   */
/* one node in its measured-performance table; it gives no scaling scheme. Reading used here:  */
/* all three expert projections run on E4M3 operands, each weight row (output feature) and    */
/* each activation row (a token row of x, a row of H) carrying one fp32 scale (amax / 448).    */
/*                                                                                              */
/* E4M3 as the OCP 8-bit floating point format defines it: sign, 4 exponent bits (bias 7),      */
/* 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; S.1111.111 is NaN; there is no  */
/* infinity; the largest finite magnitude is 448 (1.110b * 2^8).                                */
/* ------------------------------------------------------------------------------------------ */

double oracle_e4m3_to_double(uint8_t c) {
    const int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* Nearest E4M3 value of v, ties to the even mantissa; finite magnitudes above 448 give 448
 * (saturation), NaN gives the NaN code. The sign of v is kept, zero included. */
uint8_t oracle_float_to_e4m3(float v) {
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    int code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal spacing 2^-9; a count of 8 is the smallest normal, whose code is also 8 */
        code = (int)nearbyint(a * 512.0);
    } else {
        int ex;
        frexp(a, &ex);            /* a = f * 2^ex, f in [0.5, 1) */
        int e = ex - 1;           /* a in [2^e, 2^(e+1)), e in -6..8 */
        double q = nearbyint(ldexp(a, 3 - e));   /* mantissa steps of 2^(e-3): q in [8, 16] */
        if (q == 16.0) {
            e += 1;
            q = 8.0;
        }
        code = ((e + 7) << 3) | ((int)q - 8);
    }
    return sign | (uint8_t)code;
}

/* Row-wise quantisation of a bf16 matrix [R, C]: amax = max_k |x_k|; s = amax / 448 as one fp32
 * division (s = 1 for an all-zero row); q_k = E4M3(x_k / s) with x_k / s one fp32 division.
 * Then x_k ~ s * q_k. */
void oracle_quantize_rows_e4m3(const uint16_t* src, int64_t R, int64_t C, uint8_t* dst,
                               float* scale) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < C; ++k) {
            const float a = fabsf((float)bf16_to_double(src[r * C + k]));
            if (a > amax) amax = a;
        }
        const float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scale[r] = s;
        for (int64_t k = 0; k < C; ++k) {
            const float q = (float)bf16_to_double(src[r * C + k]) / s;
            dst[r * C + k] = oracle_float_to_e4m3(q);
        }
    }
}

/* FP8 down projection of given bf16 rows H [M, I]: each row is quantised like any other row
 * (oracle_quantize_rows_e4m3), W2q[e] holds the codes of Wd [d, I] with one scale per output
 * feature in w2_scale[e * d + i]:
 *   Y_i = bf16( sum_j (sh qh_j) (sw_i qw_ij) )   (double). */
static void down_row_fp8(const uint16_t* hrow, int64_t I, const uint8_t* w2q, const float* w2s,
                         int64_t d, uint16_t* yrow) {
    uint8_t* hq = (uint8_t*)malloc((size_t)I);
    float sh;
    oracle_quantize_rows_e4m3(hrow, 1, I, hq, &sh);
    double* hd = (double*)malloc((size_t)I * sizeof(double));
    for (int64_t j = 0; j < I; ++j) hd[j] = (double)sh * oracle_e4m3_to_double(hq[j]);
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < I; ++j) acc += hd[j] * ((double)w2s[i] * oracle_e4m3_to_double(w2q[i * I + j]));
        yrow[i] = oracle_double_to_bf16(acc);
    }
    free(hq); free(hd);
}

void oracle_expert_down_fp8(const uint16_t* h, const int32_t* row_expert, int64_t M, int64_t d,
                            int64_t I, const uint8_t* w2q, const float* w2_scale, uint16_t* y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        const int64_t e = row_expert[r];
        down_row_fp8(h + r * I, I, w2q + e * d * I, w2_scale + e * d, d, y + r * d);
    }
}

/* FP8 experts on grouped rows: row r holds the E4M3 codes xq[r, :] of its token with scale
 * sx[r]; W13q[e] = [Wg; Wu] codes [2I, d] with one scale per row in w13_scale[e * 2I + j];
 * W2q[e] codes [d, I] with one scale per row in w2_scale[e * d + i].
 *   G_j = sum_k (sx qx_k) (sg_j qg_jk),  U_j likewise   (double)
 *   H_j = bf16( G_j sigmoid(G_j) U_j ),  then the FP8 down projection of H above. */
void oracle_expert_rows_fp8(const uint8_t* xq, const float* sx, const int32_t* row_expert,
                            int64_t M, int64_t d, int64_t I, const uint8_t* w13q,
                            const float* w13_scale, const uint8_t* w2q, const float* w2_scale,
                            uint16_t* h, uint16_t* y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < M; ++r) {
        const int64_t e = row_expert[r];
        const uint8_t* wg = w13q + e * 2 * I * d;
        const uint8_t* wu = wg + I * d;
        const float* sg = w13_scale + e * 2 * I;
        const float* su = sg + I;
        double* xd = (double*)malloc((size_t)d * sizeof(double));
        uint16_t* hrow = (uint16_t*)malloc((size_t)I * sizeof(uint16_t));
        for (int64_t k = 0; k < d; ++k) xd[k] = (double)sx[r] * oracle_e4m3_to_double(xq[r * d + k]);
        for (int64_t j = 0; j < I; ++j) {
            double G = 0.0, U = 0.0;
            for (int64_t k = 0; k < d; ++k) {
                G += xd[k] * ((double)sg[j] * oracle_e4m3_to_double(wg[j * d + k]));
                U += xd[k] * ((double)su[j] * oracle_e4m3_to_double(wu[j * d + k]));
            }
            const double silu = G / (1.0 + exp(-G));
            hrow[j] = oracle_double_to_bf16(silu * U);
            if (h) h[r * I + j] = hrow[j];
        }
        down_row_fp8(hrow, I, w2q + e * d * I, w2_scale + e * d, d, y + r * d);
        free(xd); free(hrow);
    }
}

/* The layer with FP8 experts: as oracle_forward, with each token row quantised by
 * oracle_quantize_rows_e4m3 and every FFN pick computed by oracle_expert_rows_fp8. Routing and
 * the zero-computation experts use the bf16 x unchanged. */
int64_t oracle_forward_fp8(const uint16_t* x, const uint16_t* wr, const float* bias,
                           const uint8_t* w13q, const float* w13_scale, const uint8_t* w2q,
                           const float* w2_scale, int64_t T, int64_t d, int64_t N, int64_t Z,
                           int64_t K, int64_t I, uint16_t* out, float* logits, int32_t* idx,
                           float* gate, int32_t* counts, double* out_acc) {
    const int64_t E = N + Z;
    oracle_router_logits(x, wr, T, d, E, logits);
    int64_t bad = oracle_route(logits, bias, T, E, K, idx, gate, counts, NULL);
    uint8_t* xq = (uint8_t*)malloc((size_t)(T * d));
    float* sx = (float*)malloc((size_t)T * sizeof(float));
    oracle_quantize_rows_e4m3(x, T, d, xq, sx);
    for (int64_t t = 0; t < T; ++t) {
        double* acc = (double*)calloc((size_t)d, sizeof(double));
        uint16_t* yrow = (uint16_t*)malloc((size_t)d * sizeof(uint16_t));
        for (int64_t r = 0; r < K; ++r) {
            const int32_t e = idx[t * K + r];
            const double g = (double)gate[t * K + r];
            if (e < N) {
                oracle_expert_rows_fp8(xq + t * d, sx + t, &e, 1, d, I, w13q, w13_scale, w2q, w2_scale,
                                       NULL, yrow);
                for (int64_t c = 0; c < d; ++c) acc[c] += g * bf16_to_double(yrow[c]);
            } else {
                for (int64_t c = 0; c < d; ++c) acc[c] += bf16_to_double(x[t * d + c]) * g;  /* E_i(x) = x */
            }
        }
        for (int64_t c = 0; c < d; ++c) {
            out[t * d + c] = oracle_double_to_bf16(acc[c]);
            if (out_acc) out_acc[t * d + c] = acc[c];
        }
        free(acc); free(yrow);
    }
    free(xq); free(sx);
    return bad;
}

/* ------------------------------------------------------------------------------------------ */
/* Bias update (section 2.1, dynamic computation-budget control):                              */
/*   b_i <- b_i + mu * (K_e/K * 1/N - T_i/(K * T_all))   for all E = N + Z experts,            */
/* as these fp32 operations, each rounded once:                                                */
/*   a = (float)K_e / ((float)K * (float)N)                                                    */
/*   c = (float)T_i / ((float)K * (float)T_all)                                                */
/*   b_i = b_i + mu * (a - c)                                                                  */
/* ------------------------------------------------------------------------------------------ */

void oracle_bias_update(float* bias, const int32_t* counts, int64_t T_all, int64_t N, int64_t Z,
                        int64_t K, int64_t K_e, float mu) {
    const int64_t E = N + Z;
    const float kn = (float)K * (float)N;
    const float a = (float)K_e / kn;
    const float kt = (float)K * (float)T_all;
    for (int64_t i = 0; i < E; ++i) {
        const float c = (float)counts[i] / kt;
        const float diff = a - c;
        const float delta = mu * diff;
        bias[i] = bias[i] + delta;
    }
}
