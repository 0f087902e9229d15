// align_generic.cu -- CUDA-core residual subspace alignment (+ RMSNorm + quantiser).
//
// ReSpinQuant paper notes, key design 3: y = Q^T x, z = M y, x_out = x + Q z
// (M = R_sub - I_r), never forming the D x D T_hat.  Infra Quant II, QuaRot /
// Method: scale-free RMSNorm in FP32, then per-token symmetric absmax
// quantisation.
//
// This is the shape-generic path (any D % 16 == 0 up to 32768, r <= 64,
// float32 or bf16 I/O).  A CTA owns TB token rows, keeps them in shared memory
// as float32, and does the three steps with FP32 FMAs; Q is read through L1/L2
// once per CTA.  The rank-r contractions make it ALU-bound at large D; the
// tensor-core kernel takes over for the large bf16 shapes.
#include "common.cuh"
#include "kernels.h"

namespace rsq {

constexpr int kGenThreads = 256;
constexpr int kRmax = 64;

template <class IO, bool kQuant>
__global__ void __launch_bounds__(kGenThreads)
k_align_generic(const typename IO::T *x, const float *__restrict__ Q,
                const float *__restrict__ M, typename IO::T *x_out, uint8_t *__restrict__ codes,
                float *__restrict__ scales, int64_t T, int D, int r, int TB, int S, int bits,
                float eps) {
    extern __shared__ float4 smem4[];
    float *xs = reinterpret_cast<float *>(smem4);   // TB x D
    float *ys = xs + size_t(TB) * D;                // S x TB x kRmax partial projections
    float *zs = ys + size_t(S) * TB * kRmax;        // TB x kRmax
    __shared__ float red_f[kGenThreads / kWarp];
    __shared__ double red_d[kGenThreads / kWarp];

    const int tid = threadIdx.x;
    const int64_t ngroups = (T + TB - 1) / TB;
    const int seg = (D + S - 1) / S;
    const int qmax = (1 << (bits - 1)) - 1;
    const int row_bytes = D * bits / 8;

    for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
        const int64_t t0 = g * TB;
        const int nt = int(T - t0 < int64_t(TB) ? T - t0 : int64_t(TB));

        // stage the rows as float32
        for (int e = tid; e < nt * D / 8; e += blockDim.x) {
            float v[8];
            load8(x + t0 * D + size_t(e) * 8, v);
            store8(xs + size_t(e) * 8, v);
        }
        __syncthreads();

        // y = Q^T x, split into S partial sums over the D index
        for (int it = tid; it < TB * r * S; it += blockDim.x) {
            const int k = it % r;
            const int rest = it / r;
            const int tau = rest % TB;
            const int s = rest / TB;
            float acc = 0.f;
            if (tau < nt) {
                const int i0 = s * seg, i1 = min(D, i0 + seg);
                const float *xr = xs + size_t(tau) * D;
                for (int i = i0; i < i1; ++i) acc = fmaf(__ldg(Q + size_t(i) * r + k), xr[i], acc);
            }
            ys[(s * TB + tau) * kRmax + k] = acc;
        }
        __syncthreads();

        // z = M y
        for (int it = tid; it < TB * r; it += blockDim.x) {
            const int j = it % r, tau = it / r;
            float acc = 0.f;
            for (int k = 0; k < r; ++k) {
                float y = 0.f;
                for (int s = 0; s < S; ++s) y += ys[(s * TB + tau) * kRmax + k];
                acc = fmaf(__ldg(M + j * r + k), y, acc);
            }
            zs[tau * kRmax + j] = acc;
        }
        __syncthreads();

        for (int tau = 0; tau < nt; ++tau) {
            const int64_t t = t0 + tau;
            float *xr = xs + size_t(tau) * D;
            const float *z = zs + tau * kRmax;
            float mx = 0.f, ss = 0.f;
            // x_out = x + Q z
            for (int i = tid; i < D; i += blockDim.x) {
                const float *q = Q + size_t(i) * r;
                float acc = 0.f;
                for (int j = 0; j < r; ++j) acc = fmaf(__ldg(q + j), z[j], acc);
                const float v = xr[i] + acc;
                x_out[t * D + i] = IO::from_f(v);
                if (kQuant) {
                    xr[i] = v;
                    mx = fmaxf(mx, fabsf(v));
                    ss = fmaf(v, v, ss);
                }
            }
            if (!kQuant) continue;
            // RMSNorm statistics and the absmax of the normalised row:
            // max|n| = max|x_out| * rs, so the codes do not depend on rs.
            const float amax = block_max(mx, red_f);
            const double sum = block_sum(double(ss), red_d);
            const float ms = float(sum / double(D));
            const float rs = 1.0f / sqrtf(ms + eps);
            const RowQuant rq = row_quant(amax, qmax);
            uint8_t *crow = codes + t * row_bytes;
            for (int gq = tid; gq < D / 8; gq += blockDim.x) {
                int c[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) c[k] = quant_code(xr[8 * gq + k], rq, qmax);
                store_group(crow, gq, bits, c);
            }
            if (tid == 0) scales[t] = amax > 0.f ? (amax * rs) / float(qmax) : 0.f;
        }
        __syncthreads();
    }
}

template <class IO, bool kQuant>
static cudaError_t launch_typed(const void *x, const float *Q, const float *M, void *x_out,
                                uint8_t *codes, float *scales, int64_t T, int D, int r, int bits,
                                float eps, cudaStream_t st) {
    int TB = 16384 / D;
    TB = TB < 1 ? 1 : (TB > 16 ? 16 : TB);
    int S = kGenThreads / (TB * r);
    S = S < 1 ? 1 : S;
    const size_t smem = (size_t(TB) * D + size_t(S) * TB * kRmax + size_t(TB) * kRmax) * sizeof(float);
    auto kern = k_align_generic<IO, kQuant>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t ngroups = (T + TB - 1) / TB;
    const int64_t cap = int64_t(num_sms()) * 4;
    const int grid = int(ngroups < cap ? ngroups : cap);
    kern<<<grid, kGenThreads, smem, st>>>(
        static_cast<const typename IO::T *>(x), Q, M, static_cast<typename IO::T *>(x_out), codes,
        scales, T, D, r, TB, S, bits, eps);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

cudaError_t launch_align_generic(const void *x, const float *Q, const float *M, void *x_out,
                                 uint8_t *codes, float *scales, int64_t T, int D, int r,
                                 int bits, float eps, int dtype, bool quant, cudaStream_t s) {
    if (dtype == 0)
        return quant ? launch_typed<F32, true>(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, s)
                     : launch_typed<F32, false>(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, s);
    return quant ? launch_typed<BF16, true>(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, s)
                 : launch_typed<BF16, false>(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, s);
}

}  // namespace rsq
