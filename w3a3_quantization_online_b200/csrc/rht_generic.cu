// rht_generic.cu -- shape-generic randomised Hadamard transform + quantiser.
//
// Infra Quant II, QuaRot / Background: v = H_d diag(s) x / sqrt(d), with the
// Sylvester H of order d = 2^n computed by the fast Walsh-Hadamard transform,
// or H_d = H_{2^n} (x) H_m for d = 2^n m with m = 12 (Paley type I, q = 11).
// QuaRot / Method: per-token symmetric absmax quantisation.
//
// With GATE the input is the FFN's gated product SiLU(a) * b (QuaRot / Method:
// the online Hadamard on the down_proj input), formed in fp32 from the two
// projections a (x) and b as they are loaded; it is never rounded to the I/O
// type.
//
// One CTA per token row; the row lives in shared memory as float32 and the
// butterflies run in radix-16 register passes (4 stages per pass).  The
// 1/sqrt(d) factor never touches the data: codes do not depend on a positive
// row factor, and it is applied once to the scale.
#include "common.cuh"
#include "kernels.h"

namespace rsq {

constexpr int kRhtThreads = 256;

// Paley type-I Hadamard matrix of order 12 (q = 11), entries +-1: H = I + S with
// S = [[0, 1^T], [-1, J]], J[i][j] = chi(j - i), chi the quadratic character
// mod 11 (nonzero squares mod 11 are 1, 3, 4, 5, 9: bit mask 0x23A).
__host__ __device__ constexpr int paley12_entry(int i, int j) {
    return i == j ? 1
                  : (i == 0 ? 1
                            : (j == 0 ? -1 : (((0x23A >> ((j - i + 11) % 11)) & 1) ? 1 : -1)));
}

// padded shared-memory index (one float of padding per 16) against bank conflicts
__device__ __forceinline__ int pidx(int i) { return i + (i >> 4); }

template <class IO, int kM, bool GATE>
__global__ void __launch_bounds__(kRhtThreads)
k_rht_generic(const typename IO::T *__restrict__ x, const typename IO::T *__restrict__ xb,
              const int8_t *__restrict__ signs,
              uint8_t *__restrict__ codes, float *__restrict__ scales, int64_t T, int d,
              int logn, int bits) {
    extern __shared__ float4 smem4[];
    float *v = reinterpret_cast<float *>(smem4);
    __shared__ float red_f[kRhtThreads / kWarp];

    const int tid = threadIdx.x;
    const int n2 = 1 << logn;
    const int qmax = (1 << (bits - 1)) - 1;
    const int row_bytes = d * bits / 8;
    const float step_den = float(qmax) * sqrtf(float(d));

    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const typename IO::T *xr = x + t * d;
        // load (and gate), apply the random signs
        for (int e = tid; e < d / 8; e += blockDim.x) {
            float a[8];
            load8(xr + 8 * e, a);
            if (GATE) {
                float bv[8];
                load8(xb + t * d + 8 * e, bv);
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] = silu_gate(a[k], bv[k]);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) v[pidx(8 * e + k)] = signs[8 * e + k] < 0 ? -a[k] : a[k];
        }
        __syncthreads();

        // Sylvester transform of order 2^n along the stride-m index a (i = a*m + b),
        // four butterfly stages per pass held in registers
        for (int p = 0; p < logn; p += 4) {
            const int eb = min(4, logn - p);
            const int len = 1 << eb;
            const int ngrp = n2 >> eb;
            for (int it = tid; it < ngrp * kM; it += blockDim.x) {
                const int b = it % kM;
                const int gi = it / kM;
                const int lo = gi & ((1 << p) - 1);
                const int hi = gi >> p;
                const int base = (hi << (p + eb)) | lo;
                float a[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    a[j] = j < len ? v[pidx((base + (j << p)) * kM + b)] : 0.f;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    if (s < eb) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (!(j & (1 << s))) {
                                const float u = a[j], w = a[j | (1 << s)];
                                a[j] = u + w;
                                a[j | (1 << s)] = u - w;
                            }
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (j < len) v[pidx((base + (j << p)) * kM + b)] = a[j];
            }
            __syncthreads();
        }

        if (kM == 12) {
            // dense H_12 on each contiguous group of 12
            for (int gi = tid; gi < n2; gi += blockDim.x) {
                float in[12], out[12];
#pragma unroll
                for (int k = 0; k < 12; ++k) in[k] = v[pidx(gi * 12 + k)];
#pragma unroll
                for (int i = 0; i < 12; ++i) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 12; ++k) acc = paley12_entry(i, k) > 0 ? acc + in[k] : acc - in[k];
                    out[i] = acc;
                }
#pragma unroll
                for (int k = 0; k < 12; ++k) v[pidx(gi * 12 + k)] = out[k];
            }
            __syncthreads();
        }

        float mx = 0.f;
        for (int e = tid; e < d; e += blockDim.x) mx = fmaxf(mx, fabsf(v[pidx(e)]));
        const float amax = block_max(mx, red_f);
        const RowQuant rq = row_quant(amax, qmax);
        uint8_t *crow = codes + t * row_bytes;
        for (int g = tid; g < d / 8; g += blockDim.x) {
            int c[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) c[k] = quant_code(v[pidx(8 * g + k)], rq, qmax);
            store_group(crow, g, bits, c);
        }
        if (tid == 0) scales[t] = amax > 0.f ? amax / step_den : 0.f;
        __syncthreads();
    }
}

template <class IO, int kM, bool GATE>
static cudaError_t launch_typed(const void *x, const void *xb, const int8_t *signs, uint8_t *codes, float *scales,
                                int64_t T, int d, int bits, cudaStream_t st) {
    const int n2 = d / kM;
    int logn = 0;
    while ((1 << logn) < n2) ++logn;
    const size_t smem = size_t(d + d / 16 + 16) * sizeof(float);
    auto kern = k_rht_generic<IO, kM, GATE>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
    }
    const int64_t cap = int64_t(num_sms()) * 8;
    const int grid = int(T < cap ? T : cap);
    kern<<<grid, kRhtThreads, smem, st>>>(static_cast<const typename IO::T *>(x),
                                          static_cast<const typename IO::T *>(xb), signs, codes, scales, T, d,
                                          logn, bits);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

cudaError_t launch_rht_generic(const void *x, const int8_t *signs, int m, uint8_t *codes,
                               float *scales, int64_t T, int d, int bits, int dtype,
                               cudaStream_t s) {
    if (dtype == 0)
        return m == 12 ? launch_typed<F32, 12, false>(x, nullptr, signs, codes, scales, T, d, bits, s)
                       : launch_typed<F32, 1, false>(x, nullptr, signs, codes, scales, T, d, bits, s);
    return m == 12 ? launch_typed<BF16, 12, false>(x, nullptr, signs, codes, scales, T, d, bits, s)
                   : launch_typed<BF16, 1, false>(x, nullptr, signs, codes, scales, T, d, bits, s);
}

cudaError_t launch_rht_gate_generic(const void *a, const void *b, const int8_t *signs, int m, uint8_t *codes,
                                    float *scales, int64_t T, int d, int bits, int dtype, cudaStream_t s) {
    if (dtype == 0)
        return m == 12 ? launch_typed<F32, 12, true>(a, b, signs, codes, scales, T, d, bits, s)
                       : launch_typed<F32, 1, true>(a, b, signs, codes, scales, T, d, bits, s);
    return m == 12 ? launch_typed<BF16, 12, true>(a, b, signs, codes, scales, T, d, bits, s)
                   : launch_typed<BF16, 1, true>(a, b, signs, codes, scales, T, d, bits, s);
}

}  // namespace rsq
