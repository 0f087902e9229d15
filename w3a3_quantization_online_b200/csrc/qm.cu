// qm.cu -- the offline construction of the online alignment's (Q, M).
//
// ReSpinQuant paper notes, key design 2: at a residual connection the
// transition T = R_out R_in^T between two layers' rotations stays close to I;
// its deviation dT = T - I is decomposed by SVD, Q (D x r) takes the top-r left
// singular vectors, T_sub = Q^T T Q is the transition inside that subspace,
// and its polar factor U V^T, pulled back into SO(r), is R_sub; M = R_sub - I.
//
// Design: dT is never formed.  dT X = R_out (R_in^T X) - X and
// dT^T X = R_in (R_out^T X) - X are skinny products with the two input
// rotations (D x D float32, read as stored), so the workspace is a few D x p
// blocks.  The top-r left singular subspace comes from subspace iteration on
// dT dT^T + mu I with a block of p = 64 (r <= 32) or 96 (r <= 64) columns
// (mu = 1e-3 of the mean eigenvalue in the current block keeps the block at
// full rank when dT has rank below p; it moves every eigenvalue alike, so the
// leading subspace is the same), each iteration re-orthonormalised by
// CholeskyQR2, then a Rayleigh-Ritz step
// (eigenvectors of (dT^T X)^T (dT^T X)) picks the r leading directions.
// T_sub = (R_out^T Q)^T (R_in^T Q); its polar factor comes from the symmetric
// eigen-decomposition T_sub^T T_sub = V S^2 V^T (well conditioned: T_sub is
// close to a rotation): U = T_sub V S^-1, R_sub = U V^T, with the singular
// pair of the smallest singular value flipped when det(R_sub) = -1.
// All accumulation is float64 (the inputs are float32; Q and M are written as
// float32).  The small dense steps (Cholesky, Jacobi eigen-decompositions,
// the polar factor) run in one CTA each; the D-sized steps are tiled kernels.
// No atomics: the result is bitwise reproducible.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace rsq {

namespace {

constexpr int kQmThreads = 256;
constexpr int kGramRows = 128;  // rows of X per partial Gram block

// Skinny product tiles: a CTA computes 16 rows x 64 columns of C; its two halves
// of 128 threads take the two halves of the K range (D / 2 each) and add their
// partial sums at the end in a fixed order (no atomics).  A half stages K steps
// of 32 through two shared buffers (the next step's tiles are loaded into
// registers while the current one is multiplied); a thread holds 2 x 4 outputs.
constexpr int kGemmBM = 16, kGemmBN = 64, kGemmBK = 32;
constexpr int kGemmThreads = 256;
constexpr int kGemmLdA = kGemmBM + 2;                          // row stride of the A tile (doubles)
constexpr int kGemmTileA = kGemmBK * kGemmLdA, kGemmTileB = kGemmBK * kGemmBN;
constexpr int kGemmHalf = 2 * (kGemmTileA + kGemmTileB);       // doubles per half (two buffers)
constexpr size_t kGemmSmem = size_t(2) * kGemmHalf * 8;

// C[i][c] = sum_j op(A)[i][j] B[j][c] (- S[i][c]) (+ mu P[i][c]), A D x D
// float32 row-major (op(A) = A or A^T), B, C, S, P D x ncols float64 with row
// stride ld (even, ncols <= ld), mu a device scalar.  C may be P (each element
// is read, then written, by the same thread).  D a multiple of 64.
template <bool TRANS>
__global__ void __launch_bounds__(kGemmThreads)
k_qm_gemm(const float *__restrict__ A, const double *__restrict__ B, double *C, const double *__restrict__ S,
          const double *P, const double *__restrict__ mu, int D, int ncols, int ld) {
    extern __shared__ double gsm[];
    const int tid = threadIdx.x, half = tid >> 7, t = tid & 127;
    double *sa = gsm + half * kGemmHalf;  // [buffer][k][i], row stride kGemmLdA
    double *sb = sa + 2 * kGemmTileA;     // [buffer][k][c]
    const int i0 = blockIdx.x * kGemmBM, c0 = blockIdx.y * kGemmBN;
    const int ty = t >> 4, tx = t & 15;   // rows 2 ty, 2 ty + 1; columns 2 tx + {0, 1} and 32 + 2 tx + {0, 1}
    const int steps = D / kGemmBK / 2, k_first = half * steps * kGemmBK;
    float4 ra;                            // the next step's A values (one float4 per thread)
    double2 rb[8];                        // and B values (eight pairs per thread)
    auto load = [&](int k0) {
        if (TRANS) {  // op(A)[i][k] = A[k][i]: 32 rows k of 16 contiguous i
            ra = *reinterpret_cast<const float4 *>(A + (size_t)(k0 + (t >> 2)) * D + i0 + 4 * (t & 3));
        } else {      // A[i][k]: 16 rows i of 32 contiguous k
            ra = *reinterpret_cast<const float4 *>(A + (size_t)(i0 + (t >> 3)) * D + k0 + 4 * (t & 7));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // 32 rows k of 32 column pairs: a warp reads one row
            const int idx = t + 128 * j, kk = idx >> 5, cc = 2 * (idx & 31);
            double2 v = make_double2(0.0, 0.0);
            if (c0 + cc < ncols) {
                v = *reinterpret_cast<const double2 *>(B + (size_t)(k0 + kk) * ld + c0 + cc);
                if (c0 + cc + 1 >= ncols) v.y = 0.0;
            }
            rb[j] = v;
        }
    };
    auto store = [&](int buf) {
        double *a = sa + buf * kGemmTileA;
        double *b = sb + buf * kGemmTileB;
        if (TRANS) {
            const int kk = t >> 2, ii = 4 * (t & 3);
            a[kk * kGemmLdA + ii] = double(ra.x);
            a[kk * kGemmLdA + ii + 1] = double(ra.y);
            a[kk * kGemmLdA + ii + 2] = double(ra.z);
            a[kk * kGemmLdA + ii + 3] = double(ra.w);
        } else {
            const int ii = t >> 3, kk = 4 * (t & 7);
            a[kk * kGemmLdA + ii] = double(ra.x);
            a[(kk + 1) * kGemmLdA + ii] = double(ra.y);
            a[(kk + 2) * kGemmLdA + ii] = double(ra.z);
            a[(kk + 3) * kGemmLdA + ii] = double(ra.w);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int idx = t + 128 * j;
            *reinterpret_cast<double2 *>(b + (idx >> 5) * kGemmBN + 2 * (idx & 31)) = rb[j];
        }
    };
    double acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    load(k_first);
    store(0);
    __syncthreads();
    for (int st = 0; st < steps; ++st) {
        const int cur = st & 1;
        if (st + 1 < steps) load(k_first + (st + 1) * kGemmBK);
        const double *a = sa + cur * kGemmTileA;
        const double *b = sb + cur * kGemmTileB;
#pragma unroll 8
        for (int kk = 0; kk < kGemmBK; ++kk) {
            const double2 av = *reinterpret_cast<const double2 *>(a + kk * kGemmLdA + 2 * ty);
            const double2 b0 = *reinterpret_cast<const double2 *>(b + kk * kGemmBN + 2 * tx);
            const double2 b1 = *reinterpret_cast<const double2 *>(b + kk * kGemmBN + 32 + 2 * tx);
            const double bv[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                acc[0][n] = fma(av.x, bv[n], acc[0][n]);
                acc[1][n] = fma(av.y, bv[n], acc[1][n]);
            }
        }
        if (st + 1 < steps) store(cur ^ 1);
        __syncthreads();
    }
    // the second half's partial sums through shared memory, then first + second
    double *red = gsm;  // [8][128]
    if (half == 1) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) red[(4 * m + n) * 128 + t] = acc[m][n];
    }
    __syncthreads();
    if (half == 0) {
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int i = i0 + 2 * ty + m, c = c0 + (n < 2 ? 2 * tx + n : 32 + 2 * tx + n - 2);
                if (c < ncols) {
                    double v = acc[m][n] + red[(4 * m + n) * 128 + t];
                    if (S) v -= S[(size_t)i * ld + c];
                    if (P) v = fma(*mu, P[(size_t)i * ld + c], v);
                    C[(size_t)i * ld + c] = v;
                }
            }
    }
}

// Partial cross-Gram of a block of kGramRows rows: P[blk][a][b] = sum_i X[i][a] Y[i][b]
// (p, q <= 96), the rows in order.  Rows pass through shared memory 16 at a
// time; thread (ta, tb) of a 16 x 16 grid holds the outputs a = ta + 16 m,
// b = tb + 16 n.
constexpr int kGramChunk = 16, kGramMax = 96, kGramPer = kGramMax / 16;
__global__ void __launch_bounds__(kQmThreads)
k_qm_gram(const double *__restrict__ X, const double *__restrict__ Y, double *__restrict__ P, int D, int p, int q,
          int ld) {
    __shared__ double sx[kGramChunk][kGramMax], sy[kGramChunk][kGramMax];
    const int blk = blockIdx.x, tid = threadIdx.x, ta = tid & 15, tb = tid >> 4;
    const int r0 = blk * kGramRows, r1 = min(D, r0 + kGramRows);
    double acc[kGramPer][kGramPer];
#pragma unroll
    for (int m = 0; m < kGramPer; ++m)
#pragma unroll
        for (int n = 0; n < kGramPer; ++n) acc[m][n] = 0.0;
    for (int c0 = r0; c0 < r1; c0 += kGramChunk) {
        const int rows = min(kGramChunk, r1 - c0);
        for (int e = tid; e < rows * p; e += kQmThreads) sx[e / p][e % p] = X[(size_t)(c0 + e / p) * ld + e % p];
        for (int e = tid; e < rows * q; e += kQmThreads) sy[e / q][e % q] = Y[(size_t)(c0 + e / q) * ld + e % q];
        __syncthreads();
        for (int rr = 0; rr < rows; ++rr) {
#pragma unroll
            for (int m = 0; m < kGramPer; ++m) {
                if (ta + 16 * m >= p) continue;
                const double xv = sx[rr][ta + 16 * m];
#pragma unroll
                for (int n = 0; n < kGramPer; ++n)
                    if (tb + 16 * n < q) acc[m][n] = fma(xv, sy[rr][tb + 16 * n], acc[m][n]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int m = 0; m < kGramPer; ++m)
#pragma unroll
        for (int n = 0; n < kGramPer; ++n) {
            const int a = ta + 16 * m, b = tb + 16 * n;
            if (a < p && b < q) P[(size_t)blk * p * q + (size_t)a * q + b] = acc[m][n];
        }
}

// Partial sums of squares of a block of kGramRows rows of Y (D x p, row stride ld).
__global__ void __launch_bounds__(kQmThreads)
k_qm_sumsq(const double *__restrict__ Y, double *__restrict__ part, int D, int p, int ld) {
    __shared__ double red[kQmThreads];
    const int r0 = blockIdx.x * kGramRows, r1 = min(D, r0 + kGramRows);
    double s = 0.0;
    for (int e = threadIdx.x; e < (r1 - r0) * p; e += kQmThreads) {
        const double v = Y[(size_t)(r0 + e / p) * ld + e % p];
        s = fma(v, v, s);
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int h = kQmThreads / 2; h > 0; h >>= 1) {  // fixed tree
        if (threadIdx.x < h) red[threadIdx.x] += red[threadIdx.x + h];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// The shift of the iteration operator, mu = 1e-3 * ||Y||_F^2 / p (a thousandth
// of the mean eigenvalue of X^T dT dT^T X), or 1 when Y = 0 (T = I).
__global__ void k_qm_mu(const double *__restrict__ part, int nblk, int p, double *__restrict__ mu) {
    double s = 0.0;
    for (int b = 0; b < nblk; ++b) s += part[b];
    *mu = s > 0.0 ? 1e-3 * s / double(p) : 1.0;
}

// G = sum over blocks of P (fixed order).
__global__ void k_qm_gram_reduce(const double *__restrict__ P, double *__restrict__ G, int nblk, int n) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
        double s = 0.0;
        for (int b = 0; b < nblk; ++b) s += P[(size_t)b * n + e];
        G[e] = s;
    }
}

// out[i][c] = sum_j X[i][j] W[j][c], j < p (W p x q, row stride q); tri: W upper
// triangular (only j <= c).
__global__ void __launch_bounds__(kQmThreads)
k_qm_apply(const double *__restrict__ X, const double *__restrict__ W, double *__restrict__ out, int D, int p, int q,
           int ld_in, int ld_out, int tri) {
    const long long n = (long long)D * q;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        const int i = int(e / q), c = int(e % q);
        const int jmax = tri ? c + 1 : p;
        double s = 0.0;
        for (int j = 0; j < jmax; ++j) s = fma(X[(size_t)i * ld_in + j], W[(size_t)j * q + c], s);
        out[(size_t)i * ld_out + c] = s;
    }
}

// Deterministic starting block: splitmix64 of the element index, mapped to [-1, 1).
__global__ void k_qm_init(double *__restrict__ X, int D, int p, int ld) {
    const long long n = (long long)D * p;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
        uint64_t z = uint64_t(e) + 0x9E3779B97F4A7C15ull;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        X[(size_t)(e / p) * ld + e % p] = double(z >> 11) * 0x1p-52 - 1.0;
    }
}

// ---- small dense linear algebra in one CTA (n <= 128), shared-memory matrices

// Cyclic Jacobi on the symmetric n x n matrix a (row stride n): on return a is
// (nearly) diagonal and v holds the eigenvectors in its columns.  Disjoint
// pairs of one round-robin step rotate in parallel.  Fixed number of sweeps.
__device__ void qm_jacobi(double *a, double *v, int n, double *cs, int *pr) {
    const int tid = threadIdx.x;
    for (int e = tid; e < n * n; e += blockDim.x) v[e] = (e / n == e % n) ? 1.0 : 0.0;
    const int m = n + (n & 1);  // players of the round robin (one dummy when n is odd)
    __syncthreads();
    for (int sweep = 0; sweep < 12; ++sweep) {
        for (int step = 0; step < m - 1; ++step) {
            // pair k: players (k, m - 1 - k) of the rotated schedule
            for (int k = tid; k < m / 2; k += blockDim.x) {
                auto player = [&](int idx) { return idx == 0 ? 0 : 1 + (idx - 1 + step) % (m - 1); };
                int p = player(k), q = player(m - 1 - k);
                if (p > q) { const int t = p; p = q; q = t; }
                pr[2 * k] = p;
                pr[2 * k + 1] = q;
                double c = 1.0, s = 0.0;
                if (q < n) {
                    const double apq = a[p * n + q];
                    if (apq != 0.0) {
                        const double theta = (a[q * n + q] - a[p * n + p]) / (2.0 * apq);
                        const double t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                        c = 1.0 / sqrt(t * t + 1.0);
                        s = t * c;
                    }
                }
                cs[2 * k] = c;
                cs[2 * k + 1] = s;
            }
            __syncthreads();
            // columns: a <- a J, v <- v J (J rotates columns p, q of each pair)
            // (consecutive threads take different pairs of one row: the column
            // stride n would put a warp's accesses in one bank)
            for (int e = tid; e < (m / 2) * n; e += blockDim.x) {
                const int row = e / (m / 2), k = e % (m / 2);
                const int p = pr[2 * k], q = pr[2 * k + 1];
                if (q >= n) continue;
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double ap = a[row * n + p], aq = a[row * n + q];
                a[row * n + p] = c * ap - s * aq;
                a[row * n + q] = s * ap + c * aq;
                const double vp = v[row * n + p], vq = v[row * n + q];
                v[row * n + p] = c * vp - s * vq;
                v[row * n + q] = s * vp + c * vq;
            }
            __syncthreads();
            // rows: a <- J^T a
            for (int e = tid; e < (m / 2) * n; e += blockDim.x) {
                const int k = e / n, col = e % n;
                const int p = pr[2 * k], q = pr[2 * k + 1];
                if (q >= n) continue;
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double ap = a[p * n + col], aq = a[q * n + col];
                a[p * n + col] = c * ap - s * aq;
                a[q * n + col] = s * ap + c * aq;
            }
            __syncthreads();
        }
    }
}

// Order of the eigenvalues (diagonal of a) from largest to smallest, ties by index.
__device__ void qm_order_desc(const double *a, int n, int *order) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const double di = a[i * n + i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
            const double dj = a[j * n + j];
            rank += (dj > di) || (dj == di && j < i);
        }
        order[rank] = i;
    }
    __syncthreads();
}

// CHOL: G (p x p) = Rc^T Rc; out = Rc^-1 (upper triangular).  status bit 2 if G
// is not positive definite.  Two p x p shared arrays: the Cholesky factor L
// (Rc = L^T) in the lower triangle of the first, X = L^-1 in the second; a
// copy of the current column of L keeps the trailing update free of
// shared-memory bank conflicts.
__global__ void __launch_bounds__(kQmThreads) k_qm_chol_inv(const double *__restrict__ G, double *__restrict__ out,
                                                            int p, int *status) {
    extern __shared__ double sm[];
    double *L = sm, *X = sm + p * p;
    __shared__ double colj[kGramMax];
    const int tid = threadIdx.x;
    for (int e = tid; e < p * p; e += blockDim.x) {
        L[e] = G[e];
        X[e] = (e / p == e % p) ? 1.0 : 0.0;
    }
    __shared__ int bad;
    if (tid == 0) bad = 0;
    __syncthreads();
    for (int j = 0; j < p; ++j) {  // right-looking Cholesky, column j (lower triangle only)
        if (tid == 0) {
            const double d = L[j * p + j];
            if (!(d > 0.0)) bad = 1;
            L[j * p + j] = d > 0.0 ? sqrt(d) : 1.0;
        }
        __syncthreads();
        const double djj = L[j * p + j];
        for (int i = j + 1 + tid; i < p; i += blockDim.x) {
            const double lij = L[i * p + j] / djj;
            L[i * p + j] = lij;
            colj[i] = lij;
        }
        __syncthreads();
        const int w = p - j - 1;
        for (int e = tid; e < w * w; e += blockDim.x) {
            const int i = j + 1 + e / w, k = j + 1 + e % w;
            if (k <= i) L[i * p + k] -= colj[i] * colj[k];
        }
        __syncthreads();
    }
    // X = L^-1 by forward elimination on the rows of [L | I]: row k of X is
    // final once divided by L[k][k]; it is then taken from the rows below
    // (only its columns c <= k are nonzero)
    for (int k = 0; k < p; ++k) {
        const double dkk = L[k * p + k];
        for (int c = tid; c <= k; c += blockDim.x) X[k * p + c] /= dkk;
        __syncthreads();
        const int w = k + 1;
        for (int e = tid; e < (p - k - 1) * w; e += blockDim.x) {
            const int i = k + 1 + e / w, c = e % w;
            X[i * p + c] -= L[i * p + k] * X[k * p + c];
        }
        __syncthreads();
    }
    for (int e = tid; e < p * p; e += blockDim.x) {  // Rc^-1 = (L^-1)^T: entry (i, c) = X[c][i]
        const int i = e / p, c = e % p;
        out[e] = i <= c ? X[c * p + i] : 0.0;
    }
    if (tid == 0 && bad) atomicOr(status, 2);
}

// EIG: S (p x p) symmetric -> W (p x r): eigenvectors of the r largest eigenvalues.
__global__ void __launch_bounds__(kQmThreads) k_qm_top_eig(const double *__restrict__ S, double *__restrict__ W, int p,
                                                           int r) {
    extern __shared__ double sm[];
    double *a = sm, *v = sm + p * p, *cs = sm + 2 * p * p;
    int *pr = reinterpret_cast<int *>(cs + p + 2);
    int *order = pr + p + 2;
    for (int e = threadIdx.x; e < p * p; e += blockDim.x) a[e] = S[e];
    __syncthreads();
    qm_jacobi(a, v, p, cs, pr);
    qm_order_desc(a, p, order);
    for (int e = threadIdx.x; e < p * r; e += blockDim.x) {
        const int j = e / r, c = e % r;
        W[e] = v[j * p + order[c]];
    }
}

// POLAR: T_sub (r x r) -> M = R_sub - I (float32, r x r row-major) with
// R_sub = U V^T the polar factor in SO(r).
__global__ void __launch_bounds__(kQmThreads) k_qm_polar(const double *__restrict__ Ts, float *__restrict__ M, int r,
                                                         int *status) {
    extern __shared__ double sm[];
    double *t = sm, *a = sm + r * r, *v = sm + 2 * r * r, *u = sm + 3 * r * r, *rs = sm + 4 * r * r;
    double *cs = rs + r * r;
    int *pr = reinterpret_cast<int *>(cs + r + 2);
    int *order = pr + r + 2;
    __shared__ double sg[64];
    __shared__ int neg;
    const int tid = threadIdx.x;
    for (int e = tid; e < r * r; e += blockDim.x) t[e] = Ts[e];
    __syncthreads();
    for (int e = tid; e < r * r; e += blockDim.x) {  // a = T^T T
        const int i = e / r, j = e % r;
        double s = 0.0;
        for (int k = 0; k < r; ++k) s = fma(t[k * r + i], t[k * r + j], s);
        a[e] = s;
    }
    __syncthreads();
    qm_jacobi(a, v, r, cs, pr);
    qm_order_desc(a, r, order);
    for (int c = tid; c < r; c += blockDim.x) sg[c] = sqrt(fmax(a[c * r + c], 0.0));
    __syncthreads();
    for (int e = tid; e < r * r; e += blockDim.x) {  // u = T v diag(1/sigma)
        const int i = e / r, c = e % r;
        double s = 0.0;
        for (int k = 0; k < r; ++k) s = fma(t[i * r + k], v[k * r + c], s);
        u[e] = sg[c] > 0.0 ? s / sg[c] : 0.0;
    }
    __syncthreads();
    for (int e = tid; e < r * r; e += blockDim.x) {  // R = U V^T
        const int i = e / r, j = e % r;
        double s = 0.0;
        for (int k = 0; k < r; ++k) s = fma(u[i * r + k], v[j * r + k], s);
        rs[e] = s;
    }
    __syncthreads();
    // det(R) sign by Gaussian elimination with partial pivoting (one thread; r <= 64)
    if (tid == 0) {
        double *w = a;  // a is free now
        for (int e = 0; e < r * r; ++e) w[e] = rs[e];
        int sign = 1;
        for (int c = 0; c < r; ++c) {
            int piv = c;
            for (int i = c + 1; i < r; ++i)
                if (fabs(w[i * r + c]) > fabs(w[piv * r + c])) piv = i;
            if (piv != c) {
                sign = -sign;
                for (int k = 0; k < r; ++k) {
                    const double x = w[c * r + k];
                    w[c * r + k] = w[piv * r + k];
                    w[piv * r + k] = x;
                }
            }
            const double d = w[c * r + c];
            if (d < 0) sign = -sign;
            if (d == 0.0) {
                sign = 0;
                break;
            }
            for (int i = c + 1; i < r; ++i) {
                const double f = w[i * r + c] / d;
                for (int k = c; k < r; ++k) w[i * r + k] -= f * w[c * r + k];
            }
        }
        neg = sign < 0;
        if (sign == 0) atomicOr(status, 4);
    }
    __syncthreads();
    if (neg) {  // flip the singular pair of the smallest singular value
        const int cmin = order[r - 1];
        for (int e = tid; e < r * r; e += blockDim.x) {
            const int i = e / r, j = e % r;
            rs[e] -= 2.0 * u[i * r + cmin] * v[j * r + cmin];
        }
        __syncthreads();
    }
    for (int e = tid; e < r * r; e += blockDim.x) M[e] = float(rs[e] - ((e / r == e % r) ? 1.0 : 0.0));
}

__global__ void k_qm_out(const double *__restrict__ Qd, float *__restrict__ Q, int D, int r, int ld) {
    const long long n = (long long)D * r;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
        Q[e] = float(Qd[(size_t)(e / r) * ld + e % r]);
}

struct QmWork {
    double *X, *Y, *Z, *P, *G, *Wt, *mu;
    int p, nblk;
};

size_t qm_layout(int D, int r, QmWork *w, void *base) {
    const int p = r <= 32 ? 64 : 96;
    const int nblk = (D + kGramRows - 1) / kGramRows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const size_t oX = take(size_t(D) * p * 8), oY = take(size_t(D) * p * 8), oZ = take(size_t(D) * p * 8);
    const size_t oP = take(size_t(nblk) * p * p * 8), oG = take(size_t(p) * p * 8), oW = take(size_t(p) * p * 8);
    const size_t oM = take(8);
    if (w) {
        char *b = static_cast<char *>(base);
        w->X = reinterpret_cast<double *>(b + oX);
        w->Y = reinterpret_cast<double *>(b + oY);
        w->Z = reinterpret_cast<double *>(b + oZ);
        w->P = reinterpret_cast<double *>(b + oP);
        w->G = reinterpret_cast<double *>(b + oG);
        w->Wt = reinterpret_cast<double *>(b + oW);
        w->mu = reinterpret_cast<double *>(b + oM);
        w->p = p;
        w->nblk = nblk;
    }
    return off;
}

cudaError_t qm_check(int n) {
    count_launch(n);
    return cudaGetLastError();
}

}  // namespace

size_t qm_workspace_bytes(int D, int r) { return qm_layout(D, r, nullptr, nullptr); }

// ---- the variant that allocates nothing: a fixed scratch array in the
// library's device image (every GPU that loads the library holds it until the
// process exits).  Host code only ever sees the array's host-side stand-in; the
// device address comes from cudaGetSymbolAddress, once per device, with that
// device current.
namespace {
constexpr size_t kQmStaticBytes = size_t(8) << 20;  // 8 MiB: D <= 4608 at r <= 32, D <= 2816 above
static __device__ __align__(256) unsigned char g_qm_scratch[kQmStaticBytes];
}  // namespace

size_t qm_static_scratch_bytes() { return kQmStaticBytes; }

cudaError_t qm_static_scratch(void **ptr) {
    static void *addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_qm_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

bool qm_supports(int D, int r) { return D >= 64 && D <= 16384 && D % 64 == 0 && r >= 1 && r <= 64 && r <= D / 2; }

cudaError_t launch_qm_build(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M,
                            void *workspace, cudaStream_t s) {
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    QmWork w;
    qm_layout(D, r, &w, workspace);
    const int p = w.p;
    const int ew = int(std::min<long long>((long long)D * p / kQmThreads + 1, (long long)num_sms() * 8));
    const dim3 ggrid(D / kGemmBM, (p + kGemmBN - 1) / kGemmBN), rgrid(D / kGemmBM, (r + kGemmBN - 1) / kGemmBN);
    const size_t chol_smem = size_t(2) * p * p * 8;
    const size_t eig_smem = size_t(2) * p * p * 8 + size_t(p + 2) * 16 + size_t(2 * p + 4) * 4;
    const size_t pol_smem = size_t(5) * r * r * 8 + size_t(r + 2) * 16 + size_t(2 * r + 4) * 4;
    static bool configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(k_qm_chol_inv, cudaFuncAttributeMaxDynamicSharedMemorySize, int(2 * 96 * 96 * 8));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_qm_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGemmSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_qm_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGemmSmem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_qm_top_eig, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(2 * 96 * 96 * 8 + 98 * 16 + 196 * 4));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_qm_polar, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     int(5 * 64 * 64 * 8 + 66 * 16 + 132 * 4));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    // X <- orthonormal basis of the columns of X (CholeskyQR, twice)
    auto orth = [&](double *X, double *tmp) -> cudaError_t {
        for (int rep = 0; rep < 2; ++rep) {
            k_qm_gram<<<w.nblk, kQmThreads, 0, s>>>(X, X, w.P, D, p, p, p);
            k_qm_gram_reduce<<<(p * p + 255) / 256, 256, 0, s>>>(w.P, w.G, w.nblk, p * p);
            k_qm_chol_inv<<<1, kQmThreads, chol_smem, s>>>(w.G, w.Wt, p, status);
            k_qm_apply<<<ew, kQmThreads, 0, s>>>(X, w.Wt, tmp, D, p, p, p, p, 1);
            const cudaError_t e2 = qm_check(4);
            if (e2 != cudaSuccess) return e2;
            cudaMemcpyAsync(X, tmp, size_t(D) * p * 8, cudaMemcpyDeviceToDevice, s);
        }
        return cudaGetLastError();
    };
    // Y <- dT^T X = R_in (R_out^T X) - X, using Z as scratch
    auto dtT = [&](const double *X, double *Y, double *Zs) {
        k_qm_gemm<true><<<ggrid, kGemmThreads, kGemmSmem, s>>>(R_out, X, Zs, nullptr, nullptr, nullptr, D, p, p);
        k_qm_gemm<false><<<ggrid, kGemmThreads, kGemmSmem, s>>>(R_in, Zs, Y, X, nullptr, nullptr, D, p, p);
        return qm_check(2);
    };
    // X <- dT Y + mu X = R_out (R_in^T Y) - Y + mu X: the shift mu > 0 keeps the
    // block at full rank when dT has rank below p (the leading subspace does
    // not change: the spectrum only moves by mu)
    auto dt_shift = [&](const double *Y, double *X, double *Zs) {
        k_qm_sumsq<<<w.nblk, kQmThreads, 0, s>>>(Y, w.P, D, p, p);
        k_qm_mu<<<1, 1, 0, s>>>(w.P, w.nblk, p, w.mu);
        k_qm_gemm<true><<<ggrid, kGemmThreads, kGemmSmem, s>>>(R_in, Y, Zs, nullptr, nullptr, nullptr, D, p, p);
        k_qm_gemm<false><<<ggrid, kGemmThreads, kGemmSmem, s>>>(R_out, Zs, X, Y, X, w.mu, D, p, p);
        return qm_check(4);
    };
    k_qm_init<<<ew, kQmThreads, 0, s>>>(w.X, D, p, p);
    if ((e = qm_check(1)) != cudaSuccess) return e;
    if ((e = orth(w.X, w.Y)) != cudaSuccess) return e;
    for (int it = 0; it < iters; ++it) {
        if ((e = dtT(w.X, w.Y, w.Z)) != cudaSuccess) return e;
        if ((e = dt_shift(w.Y, w.X, w.Z)) != cudaSuccess) return e;
        if ((e = orth(w.X, w.Y)) != cudaSuccess) return e;
    }
    // Rayleigh-Ritz: S = (dT^T X)^T (dT^T X), top-r eigenvectors W, Q = X W (into Z)
    if ((e = dtT(w.X, w.Y, w.Z)) != cudaSuccess) return e;
    k_qm_gram<<<w.nblk, kQmThreads, 0, s>>>(w.Y, w.Y, w.P, D, p, p, p);
    k_qm_gram_reduce<<<(p * p + 255) / 256, 256, 0, s>>>(w.P, w.G, w.nblk, p * p);
    k_qm_top_eig<<<1, kQmThreads, eig_smem, s>>>(w.G, w.Wt, p, r);
    k_qm_apply<<<ew, kQmThreads, 0, s>>>(w.X, w.Wt, w.Z, D, p, r, p, p, 0);  // Q in Z (row stride p)
    if ((e = qm_check(4)) != cudaSuccess) return e;
    // T_sub = (R_out^T Q)^T (R_in^T Q)
    k_qm_gemm<true><<<rgrid, kGemmThreads, kGemmSmem, s>>>(R_out, w.Z, w.X, nullptr, nullptr, nullptr, D, r, p);
    k_qm_gemm<true><<<rgrid, kGemmThreads, kGemmSmem, s>>>(R_in, w.Z, w.Y, nullptr, nullptr, nullptr, D, r, p);
    k_qm_gram<<<w.nblk, kQmThreads, 0, s>>>(w.X, w.Y, w.P, D, r, r, p);
    k_qm_gram_reduce<<<(r * r + 255) / 256, 256, 0, s>>>(w.P, w.G, w.nblk, r * r);
    k_qm_polar<<<1, kQmThreads, pol_smem, s>>>(w.G, M, r, status);
    k_qm_out<<<ew, kQmThreads, 0, s>>>(w.Z, Q, D, r, p);
    return qm_check(6);
}

}  // namespace rsq
