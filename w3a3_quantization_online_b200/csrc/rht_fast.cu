// rht_fast.cu -- randomised Hadamard transform of order 4096 + per-token
// symmetric quantiser, bf16 input, one warp per token row.
//
// Infra Quant II, QuaRot / Background: v = H diag(s) x / sqrt(d) with the
// Sylvester H of order d = 2^12, computed as a fast Walsh-Hadamard transform
// (scholia log "QuaRot and SpinQuant", 2.2); QuaRot / Method: per-token
// symmetric absmax quantisation.
//
// The row is viewed as a 64 x 64 matrix X[a][b] (i = 64 a + b).  Because the
// Sylvester matrix factors as H_4096 = H_64 (x) H_64, the transform is
// W = H_64 X H_64: a 64-point transform along a for every column b, then along
// b for every row a.  Lane l of the warp holds columns (2l, 2l+1) in the first phase and
// rows (2l, 2l+1) in the second, so every butterfly of both phases is a packed
// two-wide fp32 add/sub (add.rn.f32x2 / sub.rn.f32x2) and, at the end, lane l
// owns the 128 contiguous outputs [128 l, 128 l + 128): the absmax is a warp
// reduction and the packed codes go out as coalesced 16-byte stores.
//
// Each warp streams its own rows through a one-row TMA buffer (8 KB,
// SWIZZLE_128B so the column-pair reads are conflict-free): the next row is
// requested as soon as the current one is in registers, so its load overlaps
// the whole transform.  The phases are joined by a transpose through the
// warp's own 16 KB fp32 buffer.  The 1/sqrt(4096) = 1/64 factor is applied to
// the scale only.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kWarps = 8;                   // warps (rows in flight) per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 1;
constexpr int kRowIn = 64 * 64 * 2;         // 8 KB bf16 row
constexpr int kRowS = 64 * 64 * 4;          // 16 KB fp32 transpose buffer
constexpr int kOffIn = 0;                                    // kWarps x kStages x 8 KB
constexpr int kOffS = kOffIn + kWarps * kStages * kRowIn;    // kWarps x 16 KB
constexpr int kOffMask = kOffS + kWarps * kRowS;             // 8 KB sign masks, [lane][row]
constexpr int kOffBar = kOffMask + 64 * 128;                 // kWarps x kStages mbarriers
constexpr int kBytes = kOffBar + kWarps * kStages * 8;
constexpr int kSmem = kBytes + 1024;

// In-place 64-point Sylvester transform of the 64 pairs v[0..63] (each pair is
// two independent transforms, one per component).
__device__ __forceinline__ void fwht64x2(float2 (&v)[64]) {
#pragma unroll
    for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if ((i & h) == 0) {
                const float2 u = v[i], w = v[i + h];
                v[i] = add2(u, w);
                v[i + h] = sub2(u, w);
            }
        }
    }
}

__device__ __forceinline__ uint32_t in_off(int a, int l) {  // (a, 2l..2l+1) in a SWIZZLE_128B 64x64 bf16 tile
    return uint32_t(a * 128 + (((l >> 2) ^ (a & 7)) << 4) + (l & 3) * 4);
}
__device__ __forceinline__ uint32_t mask_off(int l, int c) {  // rows 4c..4c+3 of lane l
    return uint32_t(l * 256 + ((c ^ (l & 15)) << 4));
}
__device__ __forceinline__ uint32_t s_off(int a, int chunk) {  // 16-byte chunk of row a of the 64x64 fp32 buffer
    return uint32_t(a * 256 + ((chunk ^ (a & 15)) << 4));
}

template <int BITS>
__device__ __forceinline__ void quant_store(const float2 (&u)[64], float amax, uint8_t *dst) {
    constexpr int qmax = (1 << (BITS - 1)) - 1;
    // Codes do not depend on a positive row factor: rows whose absmax is so
    // small that qmax / amax would overflow are first scaled by 2^64 (exact).
    const RowQuant rq = row_quant(amax, qmax);
    const bool tiny = rq.pre != 1.0f;
    const float2 inv2 = make_float2(rq.inv, rq.inv);
    const float2 mag2 = make_float2(kRoundMagic, kRoundMagic);
    // round(v * inv) via the 1.5*2^23 trick; |v| * qmax / amax <= qmax (+1 ulp),
    // so no clamp is needed and the low bits hold the code in two's complement.
    auto code_bits = [&](float2 v) {
        if (tiny) v = make_float2(v.x * rq.pre, v.y * rq.pre);
        const float2 t = fma2(v, inv2, mag2);
        return make_uint2(__float_as_uint(t.x), __float_as_uint(t.y));
    };
    uint32_t w[BITS * 4];
    if (BITS == 4) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // 8 columns -> one word per row
            uint32_t b0[4], b1[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint2 c0 = code_bits(u[8 * k + 2 * e]);
                const uint2 c1 = code_bits(u[8 * k + 2 * e + 1]);
                b0[e] = (c0.x & 0x0Fu) | ((c1.x << 4) & 0xF0u);
                b1[e] = (c0.y & 0x0Fu) | ((c1.y << 4) & 0xF0u);
            }
            w[k] = prmt(prmt(b0[0], b0[1], 0x0040u), prmt(b0[2], b0[3], 0x0040u), 0x5410u);
            w[8 + k] = prmt(prmt(b1[0], b1[1], 0x0040u), prmt(b1[2], b1[3], 0x0040u), 0x5410u);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // 32 codes per row -> 4 groups of 8 -> 3 words
            uint32_t g0[4], g1[4];
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
                uint32_t a0 = 0, a1 = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint2 c = code_bits(u[32 * k + 8 * gi + e]);
                    a0 |= (c.x & 0x7u) << (3 * e);
                    a1 |= (c.y & 0x7u) << (3 * e);
                }
                g0[gi] = a0;
                g1[gi] = a1;
            }
            w[k * 3 + 0] = g0[0] | (g0[1] << 24);
            w[k * 3 + 1] = (g0[1] >> 8) | (g0[2] << 16);
            w[k * 3 + 2] = (g0[2] >> 16) | (g0[3] << 8);
            w[6 + k * 3 + 0] = g1[0] | (g1[1] << 24);
            w[6 + k * 3 + 1] = (g1[1] >> 8) | (g1[2] << 16);
            w[6 + k * 3 + 2] = (g1[2] >> 16) | (g1[3] << 8);
        }
    }
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < BITS; ++q) d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
k_rht4096(const __grid_constant__ CUtensorMap tm_x, const int8_t *__restrict__ signs, uint8_t *__restrict__ codes,
          float *__restrict__ scales, long long T, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *sin = base + kOffIn + warp * kStages * kRowIn;
    uint8_t *ss = base + kOffS + warp * kRowS;
    uint8_t *smask = base + kOffMask;
    const uint32_t bar0 = smem_u32(base + kOffBar + warp * kStages * 8);
    int err = 0;

    // sign masks: bit 15 / bit 31 of word (l, a) flip the signs of elements
    // 64a + 2l and 64a + 2l + 1 (bf16 pairs); lane l reads rows 4c..4c+3 at once
    for (int idx = threadIdx.x; idx < 64 * 32; idx += kThreads) {
        const int a = idx >> 5, l = idx & 31;
        const int i = 64 * a + 2 * l;
        const uint32_t m = (signs[i] < 0 ? 0x8000u : 0u) | (signs[i + 1] < 0 ? 0x80000000u : 0u);
        reinterpret_cast<uint32_t *>(smask + mask_off(l, a >> 2))[a & 3] = m;
    }
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();

    const long long gw = (long long)blockIdx.x * kWarps + warp;
    const long long nw = (long long)gridDim.x * kWarps;
    constexpr int row_bytes = 4096 * BITS / 8;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            const long long t = gw + s * nw;
            if (t < T) {
                mbar_expect_tx(bar0 + 8 * s, kRowIn);
                if (!err) tma_load_3d(smem_u32(sin + s * kRowIn), &tm_x, 0, 0, int(t), bar0 + 8 * s);
            }
        }
    }
    __syncwarp();

    int it = 0;
    for (long long t = gw; t < T; t += nw, ++it) {
        const int s = 0;
        if (!mbar_wait(bar0, uint32_t(it & 1), err != 0)) err |= kErrMbarTimeout;

        // phase 1: columns (2l, 2l+1), all rows a; signs applied on the bf16 pairs
        float2 v[64];
        const uint8_t *xin = sin + s * kRowIn;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint4 mk = *reinterpret_cast<const uint4 *>(smask + mask_off(lane, c));
            const uint32_t m4[4] = {mk.x, mk.y, mk.z, mk.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int a = 4 * c + e;
                const uint32_t w = *reinterpret_cast<const uint32_t *>(xin + in_off(a, lane)) ^ m4[e];
                v[a] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
            }
        }
        __syncwarp();
        if (lane == 0) {  // the row buffer is free: request the next row now
            const long long tn = t + kStages * nw;
            if (tn < T) {
                mbar_expect_tx(bar0 + 8 * s, kRowIn);
                if (!err) tma_load_3d(smem_u32(sin + s * kRowIn), &tm_x, 0, 0, int(tn), bar0 + 8 * s);
            }
        }
        fwht64x2(v);  // along a for columns 2l, 2l+1
#pragma unroll
        for (int a = 0; a < 64; ++a)
            *reinterpret_cast<float2 *>(ss + s_off(a, lane >> 1) + (lane & 1) * 8) = v[a];
        __syncwarp();

        // phase 2: rows (2l, 2l+1), all columns b
        float2 u[64];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float4 r0 = *reinterpret_cast<const float4 *>(ss + s_off(2 * lane, c));
            const float4 r1 = *reinterpret_cast<const float4 *>(ss + s_off(2 * lane + 1, c));
            u[4 * c + 0] = make_float2(r0.x, r1.x);
            u[4 * c + 1] = make_float2(r0.y, r1.y);
            u[4 * c + 2] = make_float2(r0.z, r1.z);
            u[4 * c + 3] = make_float2(r0.w, r1.w);
        }
        __syncwarp();
        fwht64x2(u);  // along b for rows 2l, 2l+1

        float mx[8];  // independent partial maxima (short dependency chains)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fabsf(u[k].x), fabsf(u[k].y));
#pragma unroll
        for (int b = 8; b < 64; ++b) mx[b & 7] = fmaxf(mx[b & 7], fmaxf(fabsf(u[b].x), fabsf(u[b].y)));
#pragma unroll
        for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], mx[k + 4]);
        const float amax = warp_max(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
        quant_store<BITS>(u, amax, codes + t * row_bytes + lane * (BITS * 16));
        if (lane == 0) {
            constexpr int qmax = (1 << (BITS - 1)) - 1;
            scales[t] = amax > 0.f ? amax / float(qmax * 64) : 0.f;  // sqrt(4096) = 64
        }
    }
    if (__syncthreads_or(err)) drain_delay();  // a staged copy still in flight lands before the CTA exits
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(status, err);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

template <int BITS>
cudaError_t launch_bits(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                        cudaStream_t st) {
    static bool configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = k_rht4096<BITS>;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    EncodeTiledFn enc = encode_fn();
    int *status = device_status_word();
    if (!enc || !status) return cudaErrorInvalidValue;
    CUtensorMap map;
    const cuuint64_t dims[3] = {64, 64, cuuint64_t(T)};
    const cuuint64_t strides[2] = {128, 8192};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const long long rows_per_cta = kWarps;
    long long grid = (T + rows_per_cta - 1) / rows_per_cta;
    const long long cap = num_sms();
    if (grid > cap) grid = cap;
    kern<<<int(grid), kThreads, kSmem, st>>>(map, signs, codes, scales, T, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

bool rht_fast_supports(int d, int m, int dtype, int bits, long long T) {
    return d == 4096 && m == 1 && dtype == 1 && (bits == 3 || bits == 4) && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_rht_fast(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                            int bits, cudaStream_t s) {
    return bits == 4 ? launch_bits<4>(x, signs, codes, scales, T, s) : launch_bits<3>(x, signs, codes, scales, T, s);
}

}  // namespace rsq
