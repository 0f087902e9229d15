// heads.cu -- the online Hadamard transforms of attention (QuaRot).
//
// Infra Quant II, QuaRot / Method:
//  * key rotation: queries and keys are rotated per head after the position
//    transform, v = (I_{n_h} (x) H_{d_h}) diag(s) x / sqrt(d_h); the attention
//    scores do not change.  The rotated keys go to a post-RoPE cache quantised
//    per head (one symmetric absmax scale per token and head); the queries
//    stay in 16-bit.
//  * value projection: the online head-mixing product on the attention output,
//    z <- z (H_{n_h} (x) I_{d_h}), followed (as every linear-layer input) by the
//    per-token symmetric quantiser.
//
// k_head_rht: one warp per 256-column chunk of a token row.  Lane l holds the
// 8 consecutive columns 8 l .. 8 l + 7 of the chunk (16-byte loads for bf16);
// d_h is a power of two in [16, 256], so a head is d_h / 8 whole lanes of one
// chunk.  The butterflies of index bits 0-2 run inside the lane, those of the
// higher bits by xor shuffles among the head's lanes; the per-head absmax uses
// the same shuffles.  The 1/sqrt(d_h) factor is applied to the rotated values
// (rotation only) or to the scale (quantised keys: codes do not depend on a
// positive row factor).
//
// k_head_mix: one CTA per token row at a time; thread t owns JP consecutive
// columns j of every head (JP = 2, or 1 for 64 heads), i.e. JP * n_h values,
// and runs the n_h-point transform in registers.  Loads of one head are 4 or 2
// bytes per thread, contiguous over the warp.  The row absmax is a block
// reduction; the int8 codes are staged in shared memory and packed 8 at a time
// (INT4 words or INT3 24-bit groups).  The signs are read once per thread into a
// bit mask per column.
#include "common.cuh"
#include "kernels.h"

namespace rsq {

namespace {

constexpr int kHeadThreads = 256;

template <class IO>
__device__ __forceinline__ void store8_io(typename IO::T *p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8_io<F32>(float *p, const float (&v)[8]) { store8(p, v); }
template <>
__device__ __forceinline__ void store8_io<BF16>(__nv_bfloat16 *p, const float (&v)[8]) { store8(p, v); }

// MODE 0: rotated values out (x_out, may equal x).  MODE 1: codes and per-head scales.
template <class IO, int MODE>
__global__ void __launch_bounds__(kHeadThreads)
k_head_rht(const typename IO::T *x, const int8_t *__restrict__ signs, typename IO::T *x_out,
           uint8_t *__restrict__ codes, float *__restrict__ scales, long long T, int d, int log_lanes,
           int bits) {
    const int lane = threadIdx.x & 31;
    const long long warp0 = (long long)blockIdx.x * (kHeadThreads / 32) + (threadIdx.x >> 5);
    const long long nwarps = (long long)gridDim.x * (kHeadThreads / 32);
    const int nchunk = (d + 255) / 256;
    const int dh = 8 << log_lanes;
    const int n_heads = d / dh;
    const float inv_sqrt = rsqrtf(float(dh));
    const int qmax = MODE == 1 ? (1 << (bits - 1)) - 1 : 1;
    const long long row_bytes = (long long)d * bits / 8;

    for (long long w = warp0; w < T * nchunk; w += nwarps) {
        const long long t = w / nchunk;
        const int c0 = int(w % nchunk) * 256 + 8 * lane;  // first column of this lane
        const bool active = c0 < d;
        float v[8];
        if (active) {
            load8(x + t * d + c0, v);
            if (signs) {
                const uint2 sw = *reinterpret_cast<const uint2 *>(signs + c0);
                const uint32_t sb[2] = {sw.x, sw.y};
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (int8_t(sb[k >> 2] >> (8 * (k & 3))) < 0) v[k] = -v[k];
            }
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = 0.f;
        }
        // index bits 0-2: inside the lane
#pragma unroll
        for (int h = 1; h < 8; h <<= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (!(k & h)) {
                    const float a = v[k], b = v[k | h];
                    v[k] = a + b;
                    v[k | h] = a - b;
                }
        // higher index bits: the head's lanes (the upper partner forms partner - own)
        for (int m = 1; m < (1 << log_lanes); m <<= 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float o = __shfl_xor_sync(0xFFFFFFFFu, v[k], m);
                v[k] = upper ? o - v[k] : v[k] + o;
            }
        }
        if (MODE == 0) {
            if (active) {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] *= inv_sqrt;
                store8_io<IO>(x_out + t * d + c0, v);
            }
        } else {
            float am = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) am = fmaxf(am, fabsf(v[k]));
            for (int m = 1; m < (1 << log_lanes); m <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, m));
            if (active) {
                const RowQuant rq = row_quant(am, qmax);
                int c[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) c[k] = quant_code(v[k], rq, qmax);
                store_group(codes + t * row_bytes, c0 / 8, bits, c);
                if ((lane & ((1 << log_lanes) - 1)) == 0)
                    scales[t * n_heads + c0 / dh] = am > 0.f ? am * inv_sqrt / float(qmax) : 0.f;
            }
        }
    }
}

template <class IO, int NH, int JP>
__global__ void __launch_bounds__(kHeadThreads)
k_head_mix(const typename IO::T *__restrict__ x, const int8_t *__restrict__ signs, uint8_t *__restrict__ codes,
           float *__restrict__ scales, long long T, int dh, int bits) {
    extern __shared__ int8_t sq[];  // d int8 codes of the current row
    __shared__ float red[kHeadThreads / 32];
    const int tid = threadIdx.x;
    const int d = NH * dh;
    const int j0 = JP * tid;  // first column within a head
    const bool own = j0 < dh;
    const int qmax = (1 << (bits - 1)) - 1;
    const long long row_bytes = (long long)d * bits / 8;
    const float inv_sqrt = rsqrtf(float(NH));
    // this thread's signs (the same for every row) as bit masks, one per column
    uint64_t neg[JP];
#pragma unroll
    for (int q = 0; q < JP; ++q) {
        neg[q] = 0;
        if (own && signs)
#pragma unroll
            for (int h = 0; h < NH; ++h)
                if (signs[h * dh + j0 + q] < 0) neg[q] |= uint64_t(1) << h;
    }

    for (long long t = blockIdx.x; t < T; t += gridDim.x) {
        float v[NH][JP];
        if (own) {
            const typename IO::T *xr = x + t * d + j0;
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int q = 0; q < JP; ++q) {
                    const float f = IO::to_f(xr[h * dh + q]);
                    v[h][q] = (neg[q] >> h) & 1 ? -f : f;
                }
        } else {
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int q = 0; q < JP; ++q) v[h][q] = 0.f;
        }
        // the NH-point Walsh-Hadamard transform along the head index
#pragma unroll
        for (int s = 1; s < NH; s <<= 1)
#pragma unroll
            for (int h = 0; h < NH; ++h)
                if (!(h & s))
#pragma unroll
                    for (int q = 0; q < JP; ++q) {
                        const float a = v[h][q], b = v[h | s][q];
                        v[h][q] = a + b;
                        v[h | s][q] = a - b;
                    }
        float am = 0.f;
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < JP; ++q) am = fmaxf(am, fabsf(v[h][q]));
        const float amax = block_max(am, red);
        const RowQuant rq = row_quant(amax, qmax);
        if (own) {
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int q = 0; q < JP; ++q) sq[h * dh + j0 + q] = int8_t(quant_code(v[h][q], rq, qmax));
        }
        __syncthreads();
        uint8_t *crow = codes + t * row_bytes;
        for (int g = tid; g < d / 8; g += blockDim.x) {
            int c[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) c[k] = sq[8 * g + k];
            store_group(crow, g, bits, c);
        }
        if (tid == 0) scales[t] = amax > 0.f ? amax * inv_sqrt / float(qmax) : 0.f;
        __syncthreads();  // sq and red are reused by the next row
    }
}

template <class IO>
cudaError_t launch_head_rht_typed(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales,
                                  long long T, int d, int n_heads, int bits, bool quant, cudaStream_t s) {
    const int dh = d / n_heads;
    int log_lanes = 0;
    while ((8 << log_lanes) < dh) ++log_lanes;
    const long long tasks = T * ((d + 255) / 256);
    const long long cap = (long long)num_sms() * 8;
    const long long blocks = (tasks + (kHeadThreads / 32) - 1) / (kHeadThreads / 32);
    const int grid = int(blocks < cap ? blocks : cap);
    using E = typename IO::T;
    if (quant)
        k_head_rht<IO, 1><<<grid, kHeadThreads, 0, s>>>(static_cast<const E *>(x), signs, nullptr, codes, scales, T,
                                                        d, log_lanes, bits);
    else
        k_head_rht<IO, 0><<<grid, kHeadThreads, 0, s>>>(static_cast<const E *>(x), signs, static_cast<E *>(x_out),
                                                        nullptr, nullptr, T, d, log_lanes, 4);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template <class IO, int NH>
cudaError_t launch_head_mix_nh(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                               int dh, int bits, cudaStream_t s) {
    constexpr int JP = NH >= 64 ? 1 : 2;
    const int threads = ((dh / JP + 31) / 32) * 32;
    const size_t smem = size_t(NH) * dh;
    auto kern = k_head_mix<IO, NH, JP>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
    }
    const long long cap = (long long)num_sms() * 16;
    const int grid = int(T < cap ? T : cap);
    kern<<<grid, threads, smem, s>>>(static_cast<const typename IO::T *>(x), signs, codes, scales, T, dh, bits);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template <class IO>
cudaError_t launch_head_mix_typed(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                                  int d, int n_heads, int bits, cudaStream_t s) {
    const int dh = d / n_heads;
    switch (n_heads) {
        case 2: return launch_head_mix_nh<IO, 2>(x, signs, codes, scales, T, dh, bits, s);
        case 4: return launch_head_mix_nh<IO, 4>(x, signs, codes, scales, T, dh, bits, s);
        case 8: return launch_head_mix_nh<IO, 8>(x, signs, codes, scales, T, dh, bits, s);
        case 16: return launch_head_mix_nh<IO, 16>(x, signs, codes, scales, T, dh, bits, s);
        case 32: return launch_head_mix_nh<IO, 32>(x, signs, codes, scales, T, dh, bits, s);
        default: return launch_head_mix_nh<IO, 64>(x, signs, codes, scales, T, dh, bits, s);
    }
}

}  // namespace

bool head_rht_supports(int d, int n_heads) {
    if (n_heads < 1 || d % n_heads) return false;
    const int dh = d / n_heads;
    return dh >= 16 && dh <= 256 && (dh & (dh - 1)) == 0;
}

bool head_mix_supports(int d, int n_heads) {
    if (n_heads < 2 || n_heads > 64 || (n_heads & (n_heads - 1)) || d % n_heads) return false;
    const int dh = d / n_heads;
    const int jp = n_heads >= 64 ? 1 : 2;
    return dh % jp == 0 && dh / jp <= kHeadThreads && d % 8 == 0;
}

cudaError_t launch_head_rht(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales,
                            long long T, int d, int n_heads, int bits, bool quant, int dtype, cudaStream_t s) {
    return dtype == 0 ? launch_head_rht_typed<F32>(x, signs, x_out, codes, scales, T, d, n_heads, bits, quant, s)
                      : launch_head_rht_typed<BF16>(x, signs, x_out, codes, scales, T, d, n_heads, bits, quant, s);
}

cudaError_t launch_head_mix(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T, int d,
                            int n_heads, int bits, int dtype, cudaStream_t s) {
    return dtype == 0 ? launch_head_mix_typed<F32>(x, signs, codes, scales, T, d, n_heads, bits, s)
                      : launch_head_mix_typed<BF16>(x, signs, codes, scales, T, d, n_heads, bits, s);
}

}  // namespace rsq
