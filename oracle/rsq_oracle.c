/*
 * rsq_oracle.c -- plain, slow, float64 CPU oracle of the online activation path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * execute this file or the library built from it; only the tests, the smoke
 * check and the bench's CPU-baseline leg do.  It shares no code, header, table
 * or constant with the CUDA path.
 *
 * Every step is written as its definition, one scalar loop per formula, with
 * no blocking, fusion or reordering beyond what the definition states.  All
 * arithmetic is IEEE double (build with -ffp-contract=off so that no fused
 * multiply-add changes a rounding).  Inputs are the exact float32/bf16 values
 * of the arrays the GPU reads, widened to double by the caller.
 *
 * Sources (web pages, cited by title and section):
 *   [RSQ]  "ReSpinQuant: Efficient Layer-Wise LLM Quantization via Subspace
 *          Residual Rotation Approximation" (paper notes), key design 2
 *          (T_hat = I + Q (R_sub - I_r) Q^T) and key design 3 (the three-step
 *          online path y = Q^T x, z = M y, x_out = x + Q z, M = R_sub - I_r).
 *   [QS]   "QuaRot and SpinQuant" (scholia log), section 1.3 (normalised 4x4
 *          Hadamard worked example, absmax/7 step) and section 2.2 (fast
 *          Walsh-Hadamard transform, O(d log d), d a power of two).
 *   [IQ2]  "Infra Quant II", QuaRot / Background (normalised Hadamard entries
 *          +-1/sqrt(d); H_d = H_{2^n} (x) H_m for d = 2^n m; randomised
 *          H diag(s)), QuaRot / Method (per-token symmetric activation
 *          quantisation, row absmax / 7, scale-free RMSNorm in FP32), and
 *          SpinQuant / Motivation (symmetric quantiser
 *          alpha = max|X| / (2^(N-1) - 1), X_Q = alpha * round(X / alpha)).
 *          QuaRot / Method also places an online Hadamard on the down_proj
 *          input, which is the FFN's gated product SiLU(gate) * up; and, in
 *          attention, a per-head Hadamard on the queries and keys after the
 *          position transform (post-RoPE key cache, quantised per head) and
 *          the head-mixing product Z (H_{n_h} (x) I) on the attention output,
 *          with (I (x) H_{d_h}) (H_{n_h} (x) I) = H_{n_h d_h} when n_h and
 *          d_h are powers of two.  The quantised activations feed an INT4
 *          GEMM whose INT32 output is turned into FP16 and multiplied by the
 *          activation's per-row scale and the weight's per-column scale.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - rounding is to nearest, ties to even (rint in the default mode);
 *   - codes are clamped to the symmetric range [-qmax, qmax];
 *   - an all-zero row gets scale 0 and all codes 0;
 *   - the randomised transform is v = H (s .* x) / sqrt(d): signs first;
 *   - Kronecker index map i = a*m + b (a < 2^n, b < m):
 *       w[a m + b] = sum_{a',b'} H_{2^n}[a,a'] H_m[b,b'] u[a' m + b'];
 *   - the order-12 matrix is Paley type I at q = 11;
 *   - RMSNorm is n = x / sqrt(mean(x^2) + eps), with no weight;
 *   - INT4 packing: element 2i in the low nibble of byte i, 2i+1 in the high
 *     nibble, two's complement; INT3 packing: 8 codes per 3 bytes, code k of a
 *     group in bits [3k, 3k+3) of the little-endian 24-bit word;
 *   - FlatQuant's Kronecker affine transform: a token row x of length
 *     n = n1 n2 is the row vector vec(X) of the n1 x n2 matrix
 *     X[a][b] = x[a n2 + b] (row-major vec), and x P with P = P1 (x) P2 is
 *     vec(P1^T X P2); the quantiser that follows is the symmetric one above
 *     (not FlatQuant's asymmetric grid, which the rest of the pages do not
 *     use), with no clipping factor.
 *
 *   [IQ2] also: FlatQuant (the Kronecker-product affine transform
 *         P = P1 (x) P2 with vec(V)(P1 (x) P2) = vec(P1^T V P2), fused with
 *         the activation quantiser in one kernel).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* threads                                                                  */
/* ------------------------------------------------------------------------ */

int ora_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Hadamard matrices                                                        */
/* ------------------------------------------------------------------------ */

/* Sylvester Hadamard matrix of order n = 2^k, entries +-1 (unnormalised),
 * built by the doubling rule H_{2l} = [[H_l, H_l], [H_l, -H_l]] starting from
 * H_1 = [1].  Row-major n x n.  [QS] 1.3 prints the normalised n = 4 case. */
int ora_sylvester(int n, double *H)
{
    if (n < 1 || (n & (n - 1))) return -1;
    H[0] = 1.0;
    for (int l = 1; l < n; l *= 2) {
        for (int i = 0; i < l; ++i) {
            for (int j = 0; j < l; ++j) {
                double h = H[(int64_t)i * n + j];
                H[(int64_t)i * n + (j + l)] = h;
                H[(int64_t)(i + l) * n + j] = h;
                H[(int64_t)(i + l) * n + (j + l)] = -h;
            }
        }
    }
    return 0;
}

static int is_prime(int q)
{
    if (q < 2) return 0;
    for (int p = 2; p * p <= q; ++p)
        if (q % p == 0) return 0;
    return 1;
}

/* Paley type-I Hadamard matrix of order q + 1 for a prime q = 3 (mod 4),
 * entries +-1.  chi is the quadratic character mod q, the Jacobsthal matrix
 * is J[i][j] = chi(j - i), S = [[0, 1^T], [-1, J]] and H = I + S.
 * [IQ2] Background: "m is the order of some known Hadamard matrix". */
int ora_paley1(int q, double *H)
{
    if (!is_prime(q) || q % 4 != 3) return -1;
    int n = q + 1;
    int *chi = (int *)calloc((size_t)q, sizeof(int));
    if (!chi) return -2;
    for (int a = 1; a < q; ++a) chi[(int)(((int64_t)a * a) % q)] = 1;
    for (int a = 1; a < q; ++a)
        if (!chi[a]) chi[a] = -1;
    chi[0] = 0;
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
            double s;
            if (i == 0 && j == 0) s = 0.0;
            else if (i == 0) s = 1.0;
            else if (j == 0) s = -1.0;
            else s = (double)chi[((j - 1) - (i - 1) + q) % q];
            H[(int64_t)i * n + j] = (i == j ? 1.0 : 0.0) + s;
        }
    free(chi);
    return 0;
}

/* In-place fast Walsh-Hadamard transform of the n = 2^k values
 * v[0], v[stride], ..., v[(n-1) stride]: v <- H_n v with the Sylvester H_n,
 * unnormalised.  [QS] 2.2: O(n log n) butterflies, n a power of two. */
void ora_fwht(int n, int64_t stride, double *v)
{
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                double a = v[(int64_t)j * stride];
                double b = v[(int64_t)(j + h) * stride];
                v[(int64_t)j * stride] = a + b;
                v[(int64_t)(j + h) * stride] = a - b;
            }
}

/* ------------------------------------------------------------------------ */
/* per-row steps                                                            */
/* ------------------------------------------------------------------------ */

/* [RSQ] key design 3: y = Q^T x (D -> r), z = M y, x_out = x + Q z.
 * Q is D x r row-major (Q[i r + k]); M is r x r row-major, z_j = sum_k M[j r + k] y_k. */
static void align_row(int D, int r, const double *x, const double *Q, const double *M,
                      double *y, double *z, double *xo)
{
    for (int k = 0; k < r; ++k) {
        double s = 0.0;
        for (int i = 0; i < D; ++i) s += Q[(int64_t)i * r + k] * x[i];
        y[k] = s;
    }
    for (int j = 0; j < r; ++j) {
        double s = 0.0;
        for (int k = 0; k < r; ++k) s += M[(int64_t)j * r + k] * y[k];
        z[j] = s;
    }
    for (int i = 0; i < D; ++i) {
        double s = 0.0;
        for (int j = 0; j < r; ++j) s += Q[(int64_t)i * r + j] * z[j];
        xo[i] = x[i] + s;
    }
}

/* [IQ2] Method / Background: RMSNorm whose scale has been folded into the next
 * weights, n = x / sqrt(mean(x^2) + eps). */
static void rmsnorm_row(int D, double eps, const double *x, double *n)
{
    double ss = 0.0;
    for (int i = 0; i < D; ++i) ss += x[i] * x[i];
    double rs = 1.0 / sqrt(ss / (double)D + eps);
    for (int i = 0; i < D; ++i) n[i] = x[i] * rs;
}

/* [IQ2] SpinQuant / Motivation, symmetric case: alpha = max|v| / (2^(N-1) - 1),
 * q = round(v / alpha) (beta = 0); [IQ2] QuaRot / Method: per token, row
 * absmax / 7 for INT4.  Codes are clamped to [-qmax, qmax]; pre receives v/alpha. */
static double quant_row(int n, int bits, const double *v, int8_t *q, double *pre)
{
    int qmax = (1 << (bits - 1)) - 1;
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        double a = fabs(v[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0) {
        for (int i = 0; i < n; ++i) {
            q[i] = 0;
            if (pre) pre[i] = 0.0;
        }
        return 0.0;
    }
    double alpha = amax / (double)qmax;
    for (int i = 0; i < n; ++i) {
        double p = v[i] / alpha;
        double c = rint(p);
        if (c > qmax) c = qmax;
        if (c < -qmax) c = -qmax;
        q[i] = (int8_t)c;
        if (pre) pre[i] = p;
    }
    return alpha;
}

/* [IQ2] Background: randomised Hadamard v = H_d diag(s) x / sqrt(d), with
 * H_d = H_{2^n} (x) H_m when d = 2^n m.  The 2^n-point transform runs along
 * stride m, then the dense m x m matrix acts on each contiguous group of m. */
static void rht_row(int d, int m, const double *Hm, const double *x, const int8_t *s,
                    double *u, double *w)
{
    int n2 = d / m;
    for (int i = 0; i < d; ++i) u[i] = (double)s[i] * x[i];
    for (int b = 0; b < m; ++b) ora_fwht(n2, m, u + b);
    for (int a = 0; a < n2; ++a)
        for (int b = 0; b < m; ++b) {
            double acc = 0.0;
            for (int bp = 0; bp < m; ++bp) acc += Hm[b * m + bp] * u[(int64_t)a * m + bp];
            w[(int64_t)a * m + b] = acc;
        }
    double c = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i) w[i] = w[i] * c;
}

static void pack_int4_row(int n, const int8_t *q, uint8_t *out)
{
    for (int i = 0; i < n / 2; ++i)
        out[i] = (uint8_t)(((unsigned)q[2 * i] & 0xFu) | (((unsigned)q[2 * i + 1] & 0xFu) << 4));
}

static void pack_int3_row(int n, const int8_t *q, uint8_t *out)
{
    for (int g = 0; g < n / 8; ++g) {
        uint32_t word = 0;
        for (int k = 0; k < 8; ++k) word |= ((uint32_t)q[8 * g + k] & 7u) << (3 * k);
        out[3 * g + 0] = (uint8_t)(word & 0xFFu);
        out[3 * g + 1] = (uint8_t)((word >> 8) & 0xFFu);
        out[3 * g + 2] = (uint8_t)((word >> 16) & 0xFFu);
    }
}

/* [IQ2] QuaRot / Method: the down_proj input is the gated FFN product
 * g = SiLU(a) * b, SiLU(a) = a / (1 + exp(-a)) (a = gate projection, b = up
 * projection).  Computed in double from the exact input values. */
static void silu_gate_row(int d, const double *a, const double *b, double *g)
{
    for (int i = 0; i < d; ++i) g[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
}

/* ------------------------------------------------------------------------ */
/* exported batched entry points (OpenMP over independent token rows)       */
/* ------------------------------------------------------------------------ */

int ora_residual_align(int64_t T, int D, int r, const double *x, const double *Q,
                       const double *M, double *xo)
{
    int err = 0;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)r);
        double *z = (double *)malloc(sizeof(double) * (size_t)r);
        if (!y || !z) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t)
                align_row(D, r, x + t * D, Q, M, y, z, xo + t * D);
        }
        free(y);
        free(z);
    }
    return err;
}

int ora_rmsnorm(int64_t T, int D, double eps, const double *x, double *n)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) rmsnorm_row(D, eps, x + t * D, n + t * D);
    return 0;
}

int ora_quant_sym(int64_t T, int n, int bits, const double *v, int8_t *q, double *alpha, double *pre)
{
    if (bits < 2 || bits > 8) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        alpha[t] = quant_row(n, bits, v + t * n, q + t * n, pre ? pre + t * n : NULL);
    return 0;
}

int ora_rht(int64_t T, int d, int m, const double *Hm, const double *x, const int8_t *s, double *v)
{
    if (m < 1 || d % m) return -1;
    int n2 = d / m;
    if (n2 & (n2 - 1)) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
        if (!u) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) rht_row(d, m, Hm, x + t * d, s, u, v + t * d);
        }
        free(u);
    }
    return err;
}

int ora_pack(int64_t T, int n, int bits, const int8_t *q, uint8_t *out)
{
    if (bits == 4 && n % 2 == 0) {
        for (int64_t t = 0; t < T; ++t) pack_int4_row(n, q + t * n, out + t * (n / 2));
        return 0;
    }
    if (bits == 3 && n % 8 == 0) {
        for (int64_t t = 0; t < T; ++t) pack_int3_row(n, q + t * n, out + t * (3 * n / 8));
        return 0;
    }
    return -1;
}

/* Full align -> RMSNorm -> quantise -> pack pipeline, one row at a time.
 * xo (T x D), q (T x D), codes (T x D bits / 8), scales (T) are outputs; pre may be NULL. */
int ora_align_norm_quant(int64_t T, int D, int r, int bits, double eps, const double *x,
                         const double *Q, const double *M, double *xo, int8_t *q,
                         uint8_t *codes, double *scales, double *pre)
{
    if ((bits != 3 && bits != 4) || (D * bits) % 8 || (bits == 3 && D % 8)) return -1;
    int err = 0;
    int row_bytes = D * bits / 8;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)r);
        double *z = (double *)malloc(sizeof(double) * (size_t)r);
        double *nrm = (double *)malloc(sizeof(double) * (size_t)D);
        if (!y || !z || !nrm) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                align_row(D, r, x + t * D, Q, M, y, z, xo + t * D);
                rmsnorm_row(D, eps, xo + t * D, nrm);
                scales[t] = quant_row(D, bits, nrm, q + t * D, pre ? pre + t * D : NULL);
                if (bits == 4) pack_int4_row(D, q + t * D, codes + t * row_bytes);
                else pack_int3_row(D, q + t * D, codes + t * row_bytes);
            }
        }
        free(y);
        free(z);
        free(nrm);
    }
    return err;
}

/* Randomised Hadamard -> quantise -> pack (no normalisation). */
int ora_rht_quant(int64_t T, int d, int m, int bits, const double *Hm, const double *x,
                  const int8_t *s, int8_t *q, uint8_t *codes, double *scales, double *pre)
{
    if ((bits != 3 && bits != 4) || (d * bits) % 8 || (bits == 3 && d % 8)) return -1;
    if (m < 1 || d % m) return -1;
    int n2 = d / m;
    if (n2 & (n2 - 1)) return -1;
    int err = 0;
    int row_bytes = d * bits / 8;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
        double *v = (double *)malloc(sizeof(double) * (size_t)d);
        if (!u || !v) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                rht_row(d, m, Hm, x + t * d, s, u, v);
                scales[t] = quant_row(d, bits, v, q + t * d, pre ? pre + t * d : NULL);
                if (bits == 4) pack_int4_row(d, q + t * d, codes + t * row_bytes);
                else pack_int3_row(d, q + t * d, codes + t * row_bytes);
            }
        }
        free(u);
        free(v);
    }
    return err;
}

int ora_silu_gate(int64_t T, int d, const double *a, const double *b, double *g)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) silu_gate_row(d, a + t * d, b + t * d, g + t * d);
    return 0;
}

/* Gated FFN product -> randomised Hadamard -> quantise -> pack: the down_proj
 * input path with the gate fused (the product is never rounded to the I/O
 * type).  Same outputs as ora_rht_quant on x = SiLU(a) * b. */
int ora_rht_quant_gate(int64_t T, int d, int m, int bits, const double *Hm, const double *a,
                       const double *b, const int8_t *s, int8_t *q, uint8_t *codes, double *scales,
                       double *pre)
{
    if ((bits != 3 && bits != 4) || (d * bits) % 8 || (bits == 3 && d % 8)) return -1;
    if (m < 1 || d % m) return -1;
    int n2 = d / m;
    if (n2 & (n2 - 1)) return -1;
    int err = 0;
    int row_bytes = d * bits / 8;
#pragma omp parallel
    {
        double *g = (double *)malloc(sizeof(double) * (size_t)d);
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
        double *v = (double *)malloc(sizeof(double) * (size_t)d);
        if (!g || !u || !v) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                silu_gate_row(d, a + t * d, b + t * d, g);
                rht_row(d, m, Hm, g, s, u, v);
                scales[t] = quant_row(d, bits, v, q + t * d, pre ? pre + t * d : NULL);
                if (bits == 4) pack_int4_row(d, q + t * d, codes + t * row_bytes);
                else pack_int3_row(d, q + t * d, codes + t * row_bytes);
            }
        }
        free(g);
        free(u);
        free(v);
    }
    return err;
}


/* [IQ2] QuaRot / Method, key rotation: the per-head Hadamard of the queries and
 * keys, v = (I_{n_h} (x) H_{d_h}) diag(s) x / sqrt(d_h): head h occupies
 * columns [h d_h, (h+1) d_h) and is transformed on its own.  s may be NULL
 * (all +1). */
static void head_rht_row(int d, int n_heads, const double *x, const int8_t *s, double *v)
{
    int dh = d / n_heads;
    for (int i = 0; i < d; ++i) v[i] = (s ? (double)s[i] : 1.0) * x[i];
    for (int h = 0; h < n_heads; ++h) ora_fwht(dh, 1, v + (int64_t)h * dh);
    double c = 1.0 / sqrt((double)dh);
    for (int i = 0; i < d; ++i) v[i] = v[i] * c;
}

/* [IQ2] QuaRot / Method, value projection: the online head-mixing product on
 * the attention output, z <- z (H_{n_h} (x) I_{d_h}), here with random signs
 * first: v[h d_h + j] = sum_h' H[h][h'] s[h' d_h + j] z[h' d_h + j] / sqrt(n_h)
 * (H symmetric: the row-vector form of the pages is the same map).  s may be
 * NULL (all +1). */
static void head_mix_row(int d, int n_heads, const double *x, const int8_t *s, double *v)
{
    int dh = d / n_heads;
    for (int i = 0; i < d; ++i) v[i] = (s ? (double)s[i] : 1.0) * x[i];
    for (int j = 0; j < dh; ++j) ora_fwht(n_heads, dh, v + j);
    double c = 1.0 / sqrt((double)n_heads);
    for (int i = 0; i < d; ++i) v[i] = v[i] * c;
}

static int heads_ok(int d, int n_heads, int need_pow2_dh, int need_pow2_nh)
{
    if (n_heads < 1 || d % n_heads) return 0;
    int dh = d / n_heads;
    if (need_pow2_dh && (dh & (dh - 1))) return 0;
    if (need_pow2_nh && (n_heads & (n_heads - 1))) return 0;
    return 1;
}

int ora_head_rht(int64_t T, int d, int n_heads, const double *x, const int8_t *s, double *v)
{
    if (!heads_ok(d, n_heads, 1, 0)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) head_rht_row(d, n_heads, x + t * d, s, v + t * d);
    return 0;
}

int ora_head_mix(int64_t T, int d, int n_heads, const double *x, const int8_t *s, double *v)
{
    if (!heads_ok(d, n_heads, 0, 1)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) head_mix_row(d, n_heads, x + t * d, s, v + t * d);
    return 0;
}

/* Per-head rotation -> symmetric quantisation of each (token, head) group of
 * d_h values (the key cache is quantised per head) -> pack.  scales: T x n_heads. */
int ora_head_rht_quant(int64_t T, int d, int n_heads, int bits, const double *x, const int8_t *s,
                       int8_t *q, uint8_t *codes, double *scales, double *pre)
{
    if ((bits != 3 && bits != 4) || !heads_ok(d, n_heads, 1, 0)) return -1;
    int dh = d / n_heads;
    if ((dh * bits) % 8 || (bits == 3 && dh % 8)) return -1;
    int err = 0;
    int row_bytes = d * bits / 8;
#pragma omp parallel
    {
        double *v = (double *)malloc(sizeof(double) * (size_t)d);
        if (!v) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                head_rht_row(d, n_heads, x + t * d, s, v);
                for (int h = 0; h < n_heads; ++h)
                    scales[t * n_heads + h] = quant_row(dh, bits, v + (int64_t)h * dh, q + t * d + (int64_t)h * dh,
                                                        pre ? pre + t * d + (int64_t)h * dh : NULL);
                if (bits == 4) pack_int4_row(d, q + t * d, codes + t * row_bytes);
                else pack_int3_row(d, q + t * d, codes + t * row_bytes);
            }
        }
        free(v);
    }
    return err;
}

/* Head mixing -> per-token symmetric quantisation -> pack (the out_proj input). */
int ora_head_mix_quant(int64_t T, int d, int n_heads, int bits, const double *x, const int8_t *s,
                       int8_t *q, uint8_t *codes, double *scales, double *pre)
{
    if ((bits != 3 && bits != 4) || (d * bits) % 8 || (bits == 3 && d % 8)) return -1;
    if (!heads_ok(d, n_heads, 0, 1)) return -1;
    int err = 0;
    int row_bytes = d * bits / 8;
#pragma omp parallel
    {
        double *v = (double *)malloc(sizeof(double) * (size_t)d);
        if (!v) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                head_mix_row(d, n_heads, x + t * d, s, v);
                scales[t] = quant_row(d, bits, v, q + t * d, pre ? pre + t * d : NULL);
                if (bits == 4) pack_int4_row(d, q + t * d, codes + t * row_bytes);
                else pack_int3_row(d, q + t * d, codes + t * row_bytes);
            }
        }
        free(v);
    }
    return err;
}


/* ------------------------------------------------------------------------ */
/* the INT4 consumer GEMM                                                   */
/* ------------------------------------------------------------------------ */

/* Packed INT4 codes of one row (element 2i in the low nibble of byte i,
 * two's complement) -> integers. */
static void unpack_int4_row(int n, const uint8_t *in, int32_t *q)
{
    for (int i = 0; i < n / 2; ++i) {
        int lo = in[i] & 0xF, hi = (in[i] >> 4) & 0xF;
        q[2 * i] = lo >= 8 ? lo - 16 : lo;
        q[2 * i + 1] = hi >= 8 ? hi - 16 : hi;
    }
}

/* [IQ2] QuaRot / Method: Y = X W^T from INT4 codes.  acc[t][n] = sum_k
 * qa[t][k] qw[n][k] (exact integers), y[t][n] = acc[t][n] * sa[t] * sw[n] in
 * double: the dequantised product before its rounding to the 16-bit output.
 * ca: T x K/2 bytes, cw: N x K/2 bytes (weight row n = output column n). */
int ora_w4a4_gemm(int64_t T, int N, int K, const uint8_t *ca, const double *sa, const uint8_t *cw,
                  const double *sw, int32_t *acc, double *y)
{
    if (K % 2 || K < 2 || N < 1) return -1;
    int32_t *qw = (int32_t *)malloc(sizeof(int32_t) * (size_t)N * (size_t)K);
    if (!qw) return -2;
    for (int n = 0; n < N; ++n) unpack_int4_row(K, cw + (int64_t)n * (K / 2), qw + (int64_t)n * K);
    int err = 0;
#pragma omp parallel
    {
        int32_t *qa = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
        if (!qa) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                unpack_int4_row(K, ca + t * (K / 2), qa);
                for (int n = 0; n < N; ++n) {
                    int64_t s = 0;
                    const int32_t *w = qw + (int64_t)n * K;
                    for (int k = 0; k < K; ++k) s += (int64_t)qa[k] * w[k];
                    acc[t * N + n] = (int32_t)s;
                    y[t * N + n] = (double)s * sa[t] * sw[n];
                }
            }
        }
        free(qa);
    }
    free(qw);
    return err;
}

/* ------------------------------------------------------------------------ */
/* FlatQuant's Kronecker affine transform                                   */
/* ------------------------------------------------------------------------ */

/* [IQ2] FlatQuant: x P = vec(P1^T X P2) for P = P1 (x) P2, X the n1 x n2
 * row-major reshape of the row x.  P1 is n1 x n1, P2 is n2 x n2, row-major.
 * First Z = P1^T X (Z[i][b] = sum_a P1[a][i] X[a][b]), then V = Z P2
 * (V[i][j] = sum_b Z[i][b] P2[b][j]), v[i n2 + j] = V[i][j]. */
static void kron_affine_row(int n1, int n2, const double *P1, const double *P2, const double *x, double *z,
                            double *v)
{
    for (int i = 0; i < n1; ++i)
        for (int b = 0; b < n2; ++b) {
            double acc = 0.0;
            for (int a = 0; a < n1; ++a) acc += P1[a * n1 + i] * x[a * n2 + b];
            z[i * n2 + b] = acc;
        }
    for (int i = 0; i < n1; ++i)
        for (int j = 0; j < n2; ++j) {
            double acc = 0.0;
            for (int b = 0; b < n2; ++b) acc += z[i * n2 + b] * P2[b * n2 + j];
            v[i * n2 + j] = acc;
        }
}

/* The transform alone (tests of the index convention). */
int ora_kron_affine(int64_t T, int n1, int n2, const double *P1, const double *P2, const double *x, double *v)
{
    if (n1 < 1 || n2 < 1) return -1;
    int64_t n = (int64_t)n1 * n2;
    int err = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
        if (!z) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) kron_affine_row(n1, n2, P1, P2, x + t * n, z, v + t * n);
        }
        free(z);
    }
    return err;
}

/* [IQ2] FlatQuant: the affine transform fused with the activation quantiser,
 * Q(P1^T X P2) per token row; the per-token symmetric quantiser and packing
 * as for the other paths. */
int ora_kron_affine_quant(int64_t T, int n1, int n2, int bits, const double *P1, const double *P2,
                          const double *x, int8_t *q, uint8_t *codes, double *scales, double *pre)
{
    if (n1 < 1 || n2 < 1) return -1;
    int n = n1 * n2;
    if ((bits != 3 && bits != 4) || (n * bits) % 8 || (bits == 3 && n % 8)) return -1;
    int row_bytes = n * bits / 8;
    int err = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)n);
        double *v = (double *)malloc(sizeof(double) * (size_t)n);
        if (!z || !v) {
#pragma omp atomic write
            err = -2;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                kron_affine_row(n1, n2, P1, P2, x + t * n, z, v);
                scales[t] = quant_row(n, bits, v, q + t * n, pre ? pre + t * n : NULL);
                if (bits == 4) pack_int4_row(n, q + t * n, codes + t * row_bytes);
                else pack_int3_row(n, q + t * n, codes + t * row_bytes);
            }
        }
        free(z);
        free(v);
    }
    return err;
}
