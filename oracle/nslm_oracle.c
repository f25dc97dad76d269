/*
 * nslm_oracle.c -- the plain CPU oracle for SeedLM seed decompression and the
 * seed-matmul MoE path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  The product (the CUDA library under
 * lfsr_seeded_moe_b200/) shares no code, header, table or constant generator
 * with this file, and never calls it.
 *
 * Everything here is written for a reader checking it against the pages by eye:
 * the LFSR is stepped one bit at a time, every weight is rebuilt from its basis
 * in fp64, every dot product is a plain fp64 loop.  No blocking, no fusion, no
 * reordering beyond a parallel loop over independent output rows.
 *
 * Sources (page title, section):
 *  [BLOG]  "NanoSeedLM: LLM inference using pseudo-random numbers" (barnson.org),
 *          sections "Where this started" (block of 8 weights -> 16-bit LFSR seed,
 *          basis, int4 coefficients, shared exponent), "What I changed:
 *          September 2026" (the seed is the initial register state), "'LFSR is
 *          free'" (step the register, pull out bit fields, subtract an offset,
 *          multiply by an int4 coefficient, sum, scale; the 24 or 32 bits that
 *          follow a seed; the (q ^ 8) - 8 nibble sign extension).
 *  [K2]    "K2-Horizon-MoVA-36B-A4B -- NanoSeedLM p4mx-q4v (22.76 GB)", section
 *          "This upload" (NAME.seeds U16, NAME.coefs U16, NAME.codes U8,
 *          NAME.exp_bias I32; 100 routed experts per layer, P=4, 4.5 bits per
 *          weight, all 65,535 seeds searched).
 *  [QWEN]  "Qwen3.8-Flash-Next-NanoSeedLM-P4" model card, sections "How it
 *          works" (16-bit LFSR seed, 4 int4 coefficients and a 4-bit exponent
 *          code per 8 weights) and "The family" (P4 = 4.5 bits, P3 = 4.0 bits).
 *
 * Readings where the pages are silent (each is a definition this oracle fixes):
 *  R1 LFSR: 16-bit Fibonacci register, feedback polynomial
 *     x^16 + x^14 + x^13 + x^11 + 1.  One step shifts right by one and enters
 *     fb = s0 ^ s2 ^ s3 ^ s5 at bit 15.  (Maximal length is required by the
 *     search over all 65,535 non-zero seeds; this polynomial is primitive.)
 *  R2 The seed is the state s_0.  The basis uses the 8P states s_1 .. s_8P that
 *     follow it, i.e. 8P new register bits (24 for P=3, 32 for P=4).
 *  R3 Basis fill is column-major: U[r][j] = value(s_{1 + 8j + r}),
 *     r = 0..7 (weight in the block), j = 0..P-1 (coefficient).
 *  R4 State value: value(s) = (s - 32768) / 32768, in [-1, 1).
 *  R5 Coefficients are two's-complement nibbles, c in [-8, 7].
 *  R6 Block scale = 2^(code + exp_bias[row]), code an unsigned 4-bit number.
 *  R7 Packing (little-endian): seeds u16[N][K/8]; coefs u16[N][K/8] with c_j
 *     in bits 4j..4j+3; for P=4 the exponent codes are u8[N][K/16], block 2m in
 *     the low nibble and block 2m+1 in the high nibble; for P=3 the exponent
 *     code sits in bits 12..15 of the coefs word and there is no codes stream.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NSLMO_OK 0
#define NSLMO_ERR_ARG (-1)

/* ---------------------------------------------------------------- the LFSR */

/* [BLOG] "'LFSR is free'": one step of the 16-bit register (reading R1). */
uint16_t nslmo_lfsr_step(uint16_t s)
{
    unsigned fb = ((s >> 0) ^ (s >> 2) ^ (s >> 3) ^ (s >> 5)) & 1u;
    return (uint16_t)((s >> 1) | (fb << 15));
}

/* Number of steps until the register returns to its start state (0 for the
 * all-zero state, which never leaves itself).  Used to check maximal length. */
int32_t nslmo_lfsr_period(uint16_t seed)
{
    if (seed == 0) return 0;
    uint16_t s = nslmo_lfsr_step(seed);
    int32_t n = 1;
    while (s != seed) {
        s = nslmo_lfsr_step(s);
        ++n;
        if (n > 70000) return -1;
    }
    return n;
}

/* The states s_0 .. s_{n-1} from a seed ([BLOG] "What I changed": the seed is
 * the initial register state; reading R2). */
void nslmo_states(uint16_t seed, int32_t n, uint16_t *out)
{
    uint16_t s = seed;
    for (int32_t t = 0; t < n; ++t) {
        out[t] = s;
        s = nslmo_lfsr_step(s);
    }
}

/* ---------------------------------------------------------------- the basis */

/* [BLOG] "Where this started": run the LFSR from the seed to get an 8 x P
 * basis.  Readings R2-R4.  U is row-major: U[r * P + j]. */
void nslmo_basis(uint16_t seed, int32_t P, double *U)
{
    uint16_t s[1 + 8 * 4];
    nslmo_states(seed, 1 + 8 * P, s);
    for (int r = 0; r < 8; ++r)
        for (int j = 0; j < P; ++j)
            U[r * P + j] = ((double)s[1 + 8 * j + r] - 32768.0) / 32768.0;
}

/* Sign extension of a 4-bit two's-complement field ([BLOG] "'LFSR is free'":
 * (q ^ 8) - 8). */
static int nibble_to_int(unsigned q)
{
    return (int)((q & 0xFu) ^ 8u) - 8;
}

/* One block of 8 weights, w = 2^(code + bias) * U(seed) * c, in fp64 ([BLOG]
 * "Where this started"; [QWEN] "How it works").  Every term is a dyadic
 * rational with fewer than 53 significant bits, so the result is exact. */
void nslmo_regen_block(uint16_t seed, const int32_t *c, int32_t P, int32_t code,
                       int32_t bias, double *w8)
{
    double U[8 * 4];
    nslmo_basis(seed, P, U);
    double scale = ldexp(1.0, code + bias);
    for (int r = 0; r < 8; ++r) {
        double acc = 0.0;
        for (int j = 0; j < P; ++j) acc += U[r * P + j] * (double)c[j];
        w8[r] = scale * acc;
    }
}

/* ----------------------------------------------------- the packed streams */

/* P = 35 denotes P = 3 with 5-bit coefficients ([BLOG] "'Four bits is four
 * bits'": "Seeds, P=3, 5-bit coefficients", 4.375 bits per weight).  Reading
 * for its 35 bits per block: the seed stream as usual; the coefs word holds
 * c_0, c_1, c_2 as 5-bit two's complement in bits 0-4, 5-9, 10-14 and bit 0 of
 * the exponent code in bit 15; a codes stream u8 [N][3 K / 64] holds code bits
 * 1..3 of block b of a row at bits 3b .. 3b+2 of the row's bit string (byte
 * 3b / 8 .. , least significant bit first).  K must be a multiple of 64. */
#define NSLMO_P3C5 35

static int32_t basis_count(int32_t P) { return P == NSLMO_P3C5 ? 3 : P; }

static int fivebit_to_int(unsigned q)
{
    return (int)((q & 0x1Fu) ^ 16u) - 16;
}

/* Unpack block (i, b) of a packed matrix (reading R7, [K2] "This upload"). */
static void unpack_block(const uint16_t *seeds, const uint16_t *coefs,
                         const uint8_t *codes, int32_t nb, int32_t P, int64_t i,
                         int64_t b, uint16_t *seed, int32_t *c, int32_t *code)
{
    *seed = seeds[i * nb + b];
    unsigned q = coefs[i * nb + b];
    if (P == NSLMO_P3C5) {
        for (int j = 0; j < 3; ++j) c[j] = fivebit_to_int(q >> (5 * j));
        const uint8_t *row = codes + i * (3 * nb / 8);
        unsigned hi = 0;
        for (int t = 0; t < 3; ++t) {
            int64_t bit = 3 * b + t;
            hi |= ((row[bit / 8] >> (bit % 8)) & 1u) << t;
        }
        *code = (int32_t)(((q >> 15) & 1u) | (hi << 1));
        return;
    }
    for (int j = 0; j < P; ++j) c[j] = nibble_to_int(q >> (4 * j));
    if (P == 4) {
        unsigned byte = codes[i * (nb / 2) + b / 2];
        *code = (int32_t)((byte >> (4 * (b & 1))) & 0xFu);
    } else {
        *code = (int32_t)((q >> 12) & 0xFu);
    }
}

static int check_shape(int32_t N, int32_t K, int32_t P)
{
    if (N < 0 || K < 0 || (P != 3 && P != 4 && P != NSLMO_P3C5)) return NSLMO_ERR_ARG;
    if (K % 8 != 0) return NSLMO_ERR_ARG;
    if (P == 4 && K % 16 != 0) return NSLMO_ERR_ARG;
    if (P == NSLMO_P3C5 && K % 64 != 0) return NSLMO_ERR_ARG;
    return NSLMO_OK;
}

/* The dense fp64 weights of a packed matrix, row-major [N][K]. */
int32_t nslmo_decompress_f64(const uint16_t *seeds, const uint16_t *coefs,
                             const uint8_t *codes, const int32_t *exp_bias,
                             int32_t N, int32_t K, int32_t P, double *w_out)
{
    if (check_shape(N, K, P)) return NSLMO_ERR_ARG;
    int32_t nb = K / 8;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        for (int64_t b = 0; b < nb; ++b) {
            uint16_t seed;
            int32_t c[4], code;
            unpack_block(seeds, coefs, codes, nb, P, i, b, &seed, c, &code);
            nslmo_regen_block(seed, c, basis_count(P), code, exp_bias[i], &w_out[i * K + 8 * b]);
        }
    }
    return NSLMO_OK;
}

/* The same weights as fp32.  Returns 1 if any fp64 weight was not exactly
 * representable in fp32, else 0 (exactness holds for |bias| <= 100). */
int32_t nslmo_decompress_f32(const uint16_t *seeds, const uint16_t *coefs,
                             const uint8_t *codes, const int32_t *exp_bias,
                             int32_t N, int32_t K, int32_t P, float *w_out)
{
    if (check_shape(N, K, P)) return NSLMO_ERR_ARG;
    int32_t nb = K / 8;
    int inexact = 0;
#pragma omp parallel for schedule(static) reduction(| : inexact)
    for (int64_t i = 0; i < N; ++i) {
        for (int64_t b = 0; b < nb; ++b) {
            uint16_t seed;
            int32_t c[4], code;
            double w8[8];
            unpack_block(seeds, coefs, codes, nb, P, i, b, &seed, c, &code);
            nslmo_regen_block(seed, c, basis_count(P), code, exp_bias[i], w8);
            for (int r = 0; r < 8; ++r) {
                float f = (float)w8[r];
                if ((double)f != w8[r]) inexact = 1;
                w_out[i * K + 8 * b + r] = f;
            }
        }
    }
    return inexact;
}

/* ------------------------------------------------------------ bf16 helpers */

/* bf16 bits -> double, exactly (a bf16 is the top half of an fp32). */
double nslmo_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp64 -> bf16 with round-to-nearest, ties to even, done in exact arithmetic:
 * find the two bf16 neighbours of v and keep the nearer (the even one on a
 * tie).  Finite inputs within the bf16 range, subnormals included. */
uint16_t nslmo_f64_to_bf16(double v)
{
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    int e;
    frexp(a, &e);                    /* a = m * 2^e, m in [0.5, 1) */
    double ulp = ldexp(1.0, e - 8);  /* bf16 has 8 significant bits ... */
    if (ulp < ldexp(1.0, -133)) ulp = ldexp(1.0, -133); /* ... down to its subnormal step */
    double lo = floor(a / ulp) * ulp;
    double hi = lo + ulp;
    double pick;
    if (a - lo < hi - a) pick = lo;
    else if (a - lo > hi - a) pick = hi;
    else pick = (fmod(lo / ulp, 2.0) == 0.0) ? lo : hi;
    float f = (float)pick;            /* exact: pick has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t h = (uint16_t)(u >> 16);
    if (v < 0) h |= 0x8000u;
    return h;
}

void nslmo_f64_to_bf16_array(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nslmo_f64_to_bf16(v[i]);
}

/* ---------------------------------------------------------- seed matvec */

/* y[m][i] = sum_k W[i][k] * x[m][k], fp64, each weight rebuilt from its seed
 * as the pages require ([BLOG] "What I changed": weights are rebuilt inside
 * the matrix multiply every time; here simply in fp64). */
int32_t nslmo_seed_matvec(const uint16_t *seeds, const uint16_t *coefs,
                          const uint8_t *codes, const int32_t *exp_bias, int32_t N,
                          int32_t K, int32_t P, const uint16_t *x_bf16, int32_t M,
                          double *y)
{
    if (check_shape(N, K, P) || M < 0) return NSLMO_ERR_ARG;
    int32_t nb = K / 8;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        for (int32_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                uint16_t seed;
                int32_t c[4], code;
                double w8[8];
                unpack_block(seeds, coefs, codes, nb, P, i, b, &seed, c, &code);
                nslmo_regen_block(seed, c, basis_count(P), code, exp_bias[i], w8);
                for (int r = 0; r < 8; ++r)
                    acc += w8[r] * nslmo_bf16_to_f64(x_bf16[(int64_t)m * K + 8 * b + r]);
            }
            y[(int64_t)m * N + i] = acc;
        }
    }
    return NSLMO_OK;
}

/* Same product, with each weight first rounded to bf16 (RNE) and the input
 * given as fp64: the arithmetic of the tensor-core path, mirrored in fp64. */
int32_t nslmo_seed_matvec_bf16w(const uint16_t *seeds, const uint16_t *coefs,
                                const uint8_t *codes, const int32_t *exp_bias,
                                int32_t N, int32_t K, int32_t P, const double *x,
                                int32_t M, double *y)
{
    if (check_shape(N, K, P) || M < 0) return NSLMO_ERR_ARG;
    int32_t nb = K / 8;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        for (int32_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                uint16_t seed;
                int32_t c[4], code;
                double w8[8];
                unpack_block(seeds, coefs, codes, nb, P, i, b, &seed, c, &code);
                nslmo_regen_block(seed, c, basis_count(P), code, exp_bias[i], w8);
                for (int r = 0; r < 8; ++r)
                    acc += nslmo_bf16_to_f64(nslmo_f64_to_bf16(w8[r])) *
                           x[(int64_t)m * K + 8 * b + r];
            }
            y[(int64_t)m * N + i] = acc;
        }
    }
    return NSLMO_OK;
}

/* ------------------------------------------------------------- routing */

/* Top-k routing over E experts for each of T tokens: the k largest logits,
 * in descending order, ties to the lower expert id; the weights are the
 * softmax of the k selected logits.  (The pages route top-8 of 100 experts,
 * [BLOG] "Why K2-Horizon-MoVA"; the softmax-over-selected reading is this
 * build's, from the synthetic workload's description.) */
int32_t nslmo_route_topk(const float *logits, int32_t T, int32_t E, int32_t k,
                         int32_t *ids, double *w)
{
    if (T < 0 || E <= 0 || k <= 0 || k > E) return NSLMO_ERR_ARG;
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        unsigned char taken[4096];
        if (E > 4096) return NSLMO_ERR_ARG;
        memset(taken, 0, (size_t)E);
        for (int32_t q = 0; q < k; ++q) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: lower id wins ties */
            }
            taken[best] = 1;
            ids[t * k + q] = best;
        }
        double mx = (double)l[ids[t * k]];
        double den = 0.0;
        for (int32_t q = 0; q < k; ++q) den += exp((double)l[ids[t * k + q]] - mx);
        for (int32_t q = 0; q < k; ++q) w[t * k + q] = exp((double)l[ids[t * k + q]] - mx) / den;
    }
    return NSLMO_OK;
}

/* ---------------------------------------------------------- the expert FFN */

typedef struct {
    const uint16_t *seeds;
    const uint16_t *coefs;
    const uint8_t *codes;
    const int32_t *exp_bias;
} nslmo_stack; /* E experts stacked: expert e owns rows [e*rows, (e+1)*rows) */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* One expert matrix-vector product in fp64: rows of expert e of a stack. */
static void expert_matvec(const nslmo_stack *S, int32_t rows, int32_t K, int32_t P,
                          int32_t e, const double *x, int bf16_weights, double *y)
{
    int32_t nb = K / 8;
    int64_t ncodes = (P == 4) ? (int64_t)rows * (nb / 2) : (P == NSLMO_P3C5 ? (int64_t)rows * (3 * nb / 8) : 0);
    const uint16_t *sd = S->seeds + (int64_t)e * rows * nb;
    const uint16_t *cf = S->coefs + (int64_t)e * rows * nb;
    const uint8_t *cd = (P == 4 || P == NSLMO_P3C5) ? S->codes + (int64_t)e * ncodes : NULL;
    const int32_t *eb = S->exp_bias + (int64_t)e * rows;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        double acc = 0.0;
        for (int64_t b = 0; b < nb; ++b) {
            uint16_t seed;
            int32_t c[4], code;
            double w8[8];
            unpack_block(sd, cf, cd, nb, P, i, b, &seed, c, &code);
            nslmo_regen_block(seed, c, basis_count(P), code, eb[i], w8);
            for (int r = 0; r < 8; ++r) {
                double wr = bf16_weights ? nslmo_bf16_to_f64(nslmo_f64_to_bf16(w8[r])) : w8[r];
                acc += wr * x[8 * b + r];
            }
        }
        y[i] = acc;
    }
}

/* The routed expert FFN for T tokens ([BLOG] "Why K2-Horizon-MoVA": 100
 * routed FFN experts, top 8; gate and up, SiLU, then down; weighted sum):
 *   y_t = sum_q w[t][q] * Down[e] (SiLU(Gate[e] x_t) * (Up[e] x_t)),  e = ids[t][q].
 * mode 0: exact fp64 everywhere.
 * mode 1: the tensor-core path mirrored: weights rounded to bf16 (RNE) and
 *         the hidden activation h rounded to bf16 before the down product. */
int32_t nslmo_moe_ffn(const uint16_t *g_seeds, const uint16_t *g_coefs,
                      const uint8_t *g_codes, const int32_t *g_bias,
                      const uint16_t *u_seeds, const uint16_t *u_coefs,
                      const uint8_t *u_codes, const int32_t *u_bias,
                      const uint16_t *d_seeds, const uint16_t *d_coefs,
                      const uint8_t *d_codes, const int32_t *d_bias, int32_t E,
                      int32_t hidden, int32_t inter, int32_t P, const uint16_t *x_bf16,
                      const int32_t *ids, const double *w, int32_t T, int32_t k,
                      int32_t mode, double *y)
{
    if (check_shape(inter, hidden, P) || check_shape(hidden, inter, P)) return NSLMO_ERR_ARG;
    if (E <= 0 || T < 0 || k <= 0) return NSLMO_ERR_ARG;
    nslmo_stack G = {g_seeds, g_coefs, g_codes, g_bias};
    nslmo_stack U = {u_seeds, u_coefs, u_codes, u_bias};
    nslmo_stack D = {d_seeds, d_coefs, d_codes, d_bias};
    double *x = (double *)malloc(sizeof(double) * (size_t)hidden);
    double *g = (double *)malloc(sizeof(double) * (size_t)inter);
    double *u = (double *)malloc(sizeof(double) * (size_t)inter);
    double *h = (double *)malloc(sizeof(double) * (size_t)inter);
    double *o = (double *)malloc(sizeof(double) * (size_t)hidden);
    if (!x || !g || !u || !h || !o) {
        free(x); free(g); free(u); free(h); free(o);
        return NSLMO_ERR_ARG;
    }
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t n = 0; n < hidden; ++n) x[n] = nslmo_bf16_to_f64(x_bf16[t * hidden + n]);
        for (int32_t n = 0; n < hidden; ++n) y[t * hidden + n] = 0.0;
        for (int32_t q = 0; q < k; ++q) {
            int32_t e = ids[t * k + q];
            if (e < 0 || e >= E) {
                free(x); free(g); free(u); free(h); free(o);
                return NSLMO_ERR_ARG;
            }
            expert_matvec(&G, inter, hidden, P, e, x, mode == 1, g);
            expert_matvec(&U, inter, hidden, P, e, x, mode == 1, u);
            for (int32_t n = 0; n < inter; ++n) {
                h[n] = silu(g[n]) * u[n];
                if (mode == 1) h[n] = nslmo_bf16_to_f64(nslmo_f64_to_bf16(h[n]));
            }
            expert_matvec(&D, hidden, inter, P, e, h, mode == 1, o);
            for (int32_t n = 0; n < hidden; ++n) y[t * hidden + n] += w[t * k + q] * o[n];
        }
    }
    free(x); free(g); free(u); free(h); free(o);
    return NSLMO_OK;
}

/* ------------------------------------------------------------ seed search */

/* Solve the 4x4 (or 3x3) normal equations by Gauss-Jordan elimination with
 * partial pivoting; returns 0 if singular. */
static int solve_small(double *A, double *B, int P, int nrhs)
{
    for (int col = 0; col < P; ++col) {
        int piv = col;
        for (int r = col + 1; r < P; ++r)
            if (fabs(A[r * P + col]) > fabs(A[piv * P + col])) piv = r;
        if (fabs(A[piv * P + col]) < 1e-300) return 0;
        if (piv != col) {
            for (int q = 0; q < P; ++q) { double t = A[col * P + q]; A[col * P + q] = A[piv * P + q]; A[piv * P + q] = t; }
            for (int q = 0; q < nrhs; ++q) { double t = B[col * nrhs + q]; B[col * nrhs + q] = B[piv * nrhs + q]; B[piv * nrhs + q] = t; }
        }
        double d = A[col * P + col];
        for (int q = 0; q < P; ++q) A[col * P + q] /= d;
        for (int q = 0; q < nrhs; ++q) B[col * nrhs + q] /= d;
        for (int r = 0; r < P; ++r) {
            if (r == col) continue;
            double f = A[r * P + col];
            if (f == 0.0) continue;
            for (int q = 0; q < P; ++q) A[r * P + q] -= f * A[col * P + q];
            for (int q = 0; q < nrhs; ++q) B[r * nrhs + q] -= f * B[col * nrhs + q];
        }
    }
    return 1;
}

/* Round half to even, then clamp to the int4 range. */
static int32_t round_clamp_int4(double v)
{
    double r = nearbyint(v); /* default rounding mode: to nearest, ties to even */
    if (r < -8.0) r = -8.0;
    if (r > 7.0) r = 7.0;
    return (int32_t)r;
}

/* Brute-force seed search for one block ([BLOG] "What I changed": each block
 * walks all 65,535 seeds; [K2] "This upload": all 65,535 seeds searched).
 * For every seed in [seed_lo, seed_hi] and every code in 0..15: the
 * least-squares coefficients c = pinv(U) w / 2^(code + bias), rounded half to
 * even and clamped to [-8, 7]; the error |w - 2^(code+bias) U c|^2.  Keeps
 * the smallest error; ties go to the larger code, then the lower seed.
 *
 * d8 (may be NULL): per-weight importances, the mean square of each weight's
 * input activation ([QWEN] "How it works": the search weighted the error of
 * each weight that way).  Then err = sum_r d_r (w_r - 2^(code+bias) (U c)_r)^2
 * and, reading the pages' weighted error as the objective, the coefficients
 * are its least-squares minimiser: c = (U^T D U)^-1 U^T D w / 2^(code+bias),
 * D = diag(d), rounded and clamped as above.  d = NULL is d_r = 1, which gives
 * the unweighted search bit for bit (every product with 1.0 is exact).  The
 * operation order, fixed here, is A[a][b] = sum_r ((U_ra U_rb) d_r),
 * B[a][r] = U_ra d_r, err = sum_r d_r (e_r e_r). */
int32_t nslmo_search_block_w(const double *w8, const double *d8, int32_t P, int32_t bias,
                             int32_t seed_lo, int32_t seed_hi, int32_t *best_seed, int32_t *best_c,
                             int32_t *best_code, double *best_err)
{
    if ((P != 3 && P != 4) || seed_lo < 1 || seed_hi > 65535 || seed_lo > seed_hi)
        return NSLMO_ERR_ARG;
    double d[8];
    for (int r = 0; r < 8; ++r) d[r] = d8 ? d8[r] : 1.0;
    double err_min = INFINITY;
    int32_t s_best = -1, code_best = -1, c_best[4] = {0, 0, 0, 0};
    for (int32_t seed = seed_lo; seed <= seed_hi; ++seed) {
        double U[8 * 4];
        nslmo_basis((uint16_t)seed, P, U);
        /* pinv(U) = (U^T U)^-1 U^T, in fp64 */
        double A[16], B[4 * 8];
        for (int a = 0; a < P; ++a)
            for (int b = 0; b < P; ++b) {
                double s = 0.0;
                for (int r = 0; r < 8; ++r) s += (U[r * P + a] * U[r * P + b]) * d[r];
                A[a * P + b] = s;
            }
        for (int a = 0; a < P; ++a)
            for (int r = 0; r < 8; ++r) B[a * 8 + r] = U[r * P + a] * d[r];
        if (!solve_small(A, B, P, 8)) continue;
        double proj[4];
        for (int a = 0; a < P; ++a) {
            double s = 0.0;
            for (int r = 0; r < 8; ++r) s += B[a * 8 + r] * w8[r];
            proj[a] = s;
        }
        for (int32_t code = 15; code >= 0; --code) {
            double scale = ldexp(1.0, code + bias);
            int32_t c[4];
            for (int a = 0; a < P; ++a) c[a] = round_clamp_int4(proj[a] / scale);
            double err = 0.0;
            for (int r = 0; r < 8; ++r) {
                double v = 0.0;
                for (int a = 0; a < P; ++a) v += U[r * P + a] * (double)c[a];
                double e = w8[r] - scale * v;
                err += d[r] * (e * e);
            }
            /* strict '<': the first hit wins, and codes run from 15 down and
               seeds from low to high, so ties keep the larger code, then the
               lower seed */
            if (err < err_min) {
                err_min = err;
                s_best = seed;
                code_best = code;
                for (int a = 0; a < P; ++a) c_best[a] = c[a];
            } else if (err == err_min && code > code_best) {
                s_best = seed;
                code_best = code;
                for (int a = 0; a < P; ++a) c_best[a] = c[a];
            }
        }
    }
    *best_seed = s_best;
    *best_code = code_best;
    for (int a = 0; a < P; ++a) best_c[a] = c_best[a];
    *best_err = err_min;
    return NSLMO_OK;
}

int32_t nslmo_search_block(const double *w8, int32_t P, int32_t bias, int32_t seed_lo,
                           int32_t seed_hi, int32_t *best_seed, int32_t *best_c,
                           int32_t *best_code, double *best_err)
{
    return nslmo_search_block_w(w8, NULL, P, bias, seed_lo, seed_hi, best_seed, best_c, best_code,
                                best_err);
}
