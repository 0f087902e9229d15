// kron_affine.cu -- FlatQuant's Kronecker affine transform fused with the
// per-token symmetric quantiser.
//
// Infra Quant II, FlatQuant: a linear layer's input row x (length d = n1 n2)
// is transformed by P = P1 (x) P2, two small invertible matrices found by
// calibration; with X the n1 x n2 row-major reshape of x,
//     x P = vec(P1^T X P2),
// and one kernel loads P1 and P2 on chip, transforms each token's n1 x n2 tile
// and quantises it before anything is written back.  The quantiser is the
// per-token symmetric absmax one of the other paths (QuaRot / Method).
//
// Design: the factors are dense and arbitrary (not +-1), so an exact product
// on the bf16 tensor cores does not exist, and float32 accumulation over
// n1 + n2 terms is ~1e-5 relative -- above the 1e-6 the scales are held to.
// The two products therefore run in float64 on the CUDA cores from the exact
// float32 / bf16 inputs (every product of two float32 values is exact in
// float64), and the quantiser works on float64 values as the oracle does.
// One CTA per SM walks the token rows; P1 and P2 stay in shared memory as
// float64; per row the tile X is staged, Z = P1^T X is formed (stored
// transposed), then V = Z P2 is formed in registers, 4 x 4 outputs per thread
// (n1 n2 <= 4096 gives at most one tile of each product per thread), and the
// row's absmax, codes and scale follow.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace rsq {

namespace {

constexpr int kAffThreads = 256;

size_t affine_smem_bytes(int n1, int n2) {
    const size_t d = size_t(n1) * n2;
    return 8 * (size_t(n1) * n1 + size_t(n2) * n2 + 2 * d) + d;
}

template <typename IO, int BITS>
__global__ void __launch_bounds__(kAffThreads)
k_kron_affine_quant(const typename IO::T *__restrict__ x, const float *__restrict__ P1,
                    const float *__restrict__ P2, int n1, int n2, long long T, uint8_t *__restrict__ codes,
                    float *__restrict__ scales) {
    extern __shared__ __align__(16) double aff_smem[];
    const int d = n1 * n2, tid = threadIdx.x;
    double *p1 = aff_smem;          // n1 x n1
    double *p2 = p1 + n1 * n1;      // n2 x n2
    double *xs = p2 + n2 * n2;      // the row's tile X, n1 x n2
    double *zt = xs + d;            // Z^T: zt[b n1 + i] = Z[i][b]
    int8_t *qs = reinterpret_cast<int8_t *>(zt + d);
    __shared__ double wmax[kAffThreads / kWarp];
    for (int e = tid; e < n1 * n1; e += kAffThreads) p1[e] = double(P1[e]);
    for (int e = tid; e < n2 * n2; e += kAffThreads) p2[e] = double(P2[e]);
    // this thread's 4 x 4 tile of Z and of V: rows i0.., columns c0.. (consecutive
    // threads take consecutive row blocks, so the Z^T stores stay 2-way)
    const int tn1 = n1 >> 2, tiles = tn1 * (n2 >> 2);
    const bool mine = tid < tiles;
    const int i0 = 4 * (tid % tn1), c0 = 4 * (tid / tn1);
    constexpr int qmax = (1 << (BITS - 1)) - 1;
    const long long row_bytes = (long long)d * BITS / 8;

    for (long long t = blockIdx.x; t < T; t += gridDim.x) {
        const typename IO::T *xr = x + t * d;
        __syncthreads();  // the previous row is done with xs, zt and qs (and p1, p2 are stored)
        for (int e = tid; e < d; e += kAffThreads) xs[e] = double(IO::to_f(xr[e]));
        __syncthreads();
        if (mine) {  // Z[i][b] = sum_a P1[a][i] X[a][b]
            double acc[4][4];
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[m][k] = 0.0;
            for (int a = 0; a < n1; ++a) {
                const double2 pa = *reinterpret_cast<const double2 *>(p1 + a * n1 + i0);
                const double2 pb = *reinterpret_cast<const double2 *>(p1 + a * n1 + i0 + 2);
                const double2 xa = *reinterpret_cast<const double2 *>(xs + a * n2 + c0);
                const double2 xb = *reinterpret_cast<const double2 *>(xs + a * n2 + c0 + 2);
                const double pv[4] = {pa.x, pa.y, pb.x, pb.y}, xv[4] = {xa.x, xa.y, xb.x, xb.y};
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[m][k] = fma(pv[m], xv[k], acc[m][k]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                double *zr = zt + (c0 + k) * n1 + i0;
                *reinterpret_cast<double2 *>(zr) = make_double2(acc[0][k], acc[1][k]);
                *reinterpret_cast<double2 *>(zr + 2) = make_double2(acc[2][k], acc[3][k]);
            }
        }
        __syncthreads();
        double v[4][4];
        double amax = 0.0;
        if (mine) {  // V[i][j] = sum_b Z[i][b] P2[b][j]
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int k = 0; k < 4; ++k) v[m][k] = 0.0;
            for (int b = 0; b < n2; ++b) {
                const double2 za = *reinterpret_cast<const double2 *>(zt + b * n1 + i0);
                const double2 zb = *reinterpret_cast<const double2 *>(zt + b * n1 + i0 + 2);
                const double2 qa = *reinterpret_cast<const double2 *>(p2 + b * n2 + c0);
                const double2 qb = *reinterpret_cast<const double2 *>(p2 + b * n2 + c0 + 2);
                const double zv[4] = {za.x, za.y, zb.x, zb.y}, qv[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
                for (int m = 0; m < 4; ++m)
#pragma unroll
                    for (int k = 0; k < 4; ++k) v[m][k] = fma(zv[m], qv[k], v[m][k]);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int k = 0; k < 4; ++k) amax = fmax(amax, fabs(v[m][k]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if ((tid & (kWarp - 1)) == 0) wmax[tid / kWarp] = amax;
        __syncthreads();
        amax = wmax[0];
#pragma unroll
        for (int w = 1; w < kAffThreads / kWarp; ++w) amax = fmax(amax, wmax[w]);
        // alpha = amax / qmax, code = clamp(rint(v / alpha)): the same float64
        // operations as the oracle's quantiser
        const double alpha = amax / double(qmax);
        if (mine) {
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    double c = 0.0;
                    if (amax > 0.0) c = fmin(fmax(rint(v[m][k] / alpha), -double(qmax)), double(qmax));
                    qs[(i0 + m) * n2 + c0 + k] = int8_t(c);
                }
        }
        __syncthreads();
        uint8_t *crow = codes + t * row_bytes;
        for (int g = tid; g < d / 8; g += kAffThreads) {
            int c[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) c[k] = qs[8 * g + k];
            store_group(crow, g, BITS, c);
        }
        if (tid == 0) scales[t] = amax > 0.0 ? float(alpha) : 0.f;
    }
}

template <typename IO, int BITS>
cudaError_t launch_typed(const void *x, const float *P1, const float *P2, int n1, int n2, uint8_t *codes,
                         float *scales, long long T, cudaStream_t s) {
    static size_t configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = k_kron_affine_quant<IO, BITS>;
    const size_t smem = affine_smem_bytes(n1, n2);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (smem > configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        configured[dev] = smem;
    }
    long long grid = num_sms();
    if (grid > T) grid = T;
    kern<<<unsigned(grid), kAffThreads, smem, s>>>(static_cast<const typename IO::T *>(x), P1, P2, n1, n2, T, codes,
                                                   scales);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

// Every shape accepted here needs at most 204 KB of shared memory (n1 = 32,
// n2 = 128), inside the 227 KB a CTA may opt into on sm_100.
bool kron_affine_supports(int n1, int n2) {
    if (n1 < 4 || n2 < 4 || n1 > 128 || n2 > 128 || n1 % 4 || n2 % 4) return false;
    return n1 * n2 <= 4096;
}

cudaError_t launch_kron_affine_quant(const void *x, const float *P1, const float *P2, int n1, int n2,
                                     uint8_t *codes, float *scales, long long T, int bits, int dtype,
                                     cudaStream_t s) {
    if (dtype == 1)
        return bits == 4 ? launch_typed<BF16, 4>(x, P1, P2, n1, n2, codes, scales, T, s)
                         : launch_typed<BF16, 3>(x, P1, P2, n1, n2, codes, scales, T, s);
    return bits == 4 ? launch_typed<F32, 4>(x, P1, P2, n1, n2, codes, scales, T, s)
                     : launch_typed<F32, 3>(x, P1, P2, n1, n2, codes, scales, T, s);
}

}  // namespace rsq
