// common.cuh -- device helpers shared by the rsq kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rsq {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// I/O element types
// ---------------------------------------------------------------------------

struct F32 {
    using T = float;
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};

struct BF16 {
    using T = __nv_bfloat16;
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// Load 8 consecutive elements (16 B for bf16, 32 B for fp32) as float.
__device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void store8(float *p, const float (&v)[8]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = u;
}

// ---------------------------------------------------------------------------
// Gated FFN product SiLU(a) * b = a * sigmoid(a) * b in fp32 (the down_proj
// input), sigmoid(a) = 1 / (1 + e^-a), with CUDA's accurate expf (the fast
// exponential's relative error grows with |a|, and a row of equal gates would
// carry it straight into the scale).  For a below about -88, e^-a overflows to
// +inf and the reciprocal gives 0, the limit of the product.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float silu_gate(float a, float b) {
    return (a * __frcp_rn(1.0f + expf(-a))) * b;
}

// ---------------------------------------------------------------------------
// Quantiser: code = clamp(round_half_even(v * inv), -qmax, qmax).
// fmaf(v, inv, 1.5 * 2^23) rounds the exact product v*inv to the nearest
// integer (ties to even) because the float grid has unit spacing there; the
// integer is read back from the low mantissa bits.  Valid for |v*inv| < 2^22.
// ---------------------------------------------------------------------------

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int quant_code(float v, float inv, int qmax) {
    const int c = __float_as_int(fmaf(v, inv, kRoundMagic)) - kRoundMagicBits;
    return max(-qmax, min(qmax, c));
}

// Per-row quantiser constants.  Codes do not depend on a positive row factor,
// so a row whose absmax is so small that qmax / amax would overflow float32 is
// quantised after an exact scaling by 2^64 (pre).
struct RowQuant {
    float inv;  // qmax / (amax * pre), 0 for an all-zero row
    float pre;  // 1, or 2^64 for rows with amax < 2^-64
};

__device__ __forceinline__ RowQuant row_quant(float amax, int qmax) {
    RowQuant q;
    q.pre = amax < 0x1p-64f ? 0x1p64f : 1.0f;
    q.inv = amax > 0.f ? float(qmax) / (amax * q.pre) : 0.f;
    return q;
}

__device__ __forceinline__ int quant_code(float v, const RowQuant &q, int qmax) {
    return quant_code(v * q.pre, q.inv, qmax);
}

// ---------------------------------------------------------------------------
// Packed two-wide fp32 arithmetic (sm_100 builtins): one instruction per pair.
// a - b is computed as fma(b, -1, a): exact product, one rounding, the same
// result as a plain subtraction.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Codes of 8 consecutive values packed into one INT4 word (or 24 bits of INT3).
// round(v * inv) uses the 1.5*2^23 trick; because |v| <= amax and
// inv = qmax / amax, |v * inv| <= qmax up to one rounding of inv, so no clamp
// is needed and the low bits of the result hold the code in two's complement.
// `pre` (1, or 2^64 for rows with a tiny absmax) is applied first when `scaled`.
template <int BITS>
__device__ __forceinline__ uint32_t pack8_fast(const float (&v)[8], float inv, float pre, bool scaled) {
    const float2 inv2 = make_float2(inv, inv);
    const float2 mag2 = make_float2(kRoundMagic, kRoundMagic);
    uint32_t r[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        float2 t = make_float2(v[e], v[e + 1]);
        if (scaled) t = mul2(t, make_float2(pre, pre));
        const float2 q = fma2(t, inv2, mag2);
        r[e] = __float_as_uint(q.x);
        r[e + 1] = __float_as_uint(q.y);
    }
    if (BITS == 4) {
        // gather the low bytes of the even and of the odd elements, then byte k =
        // low nibble of r[2k] | low nibble of r[2k+1] << 4
        const uint32_t ev = prmt(prmt(r[0], r[2], 0x0040u), prmt(r[4], r[6], 0x0040u), 0x5410u);
        const uint32_t od = prmt(prmt(r[1], r[3], 0x0040u), prmt(r[5], r[7], 0x0040u), 0x5410u);
        return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    } else {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= (r[e] & 0x7u) << (3 * e);
        return w;
    }
}

// Pack 8 codes (each in [-qmax, qmax]).
__device__ __forceinline__ uint32_t pack8_int4(const int (&c)[8]) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= (uint32_t(c[k]) & 0xFu) << (4 * k);
    return w;
}

__device__ __forceinline__ uint32_t pack8_int3(const int (&c)[8]) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= (uint32_t(c[k]) & 0x7u) << (3 * k);
    return w;  // 24 significant bits
}

// Store the packed 8-code group g of a row (INT4: 4 bytes at 4g, INT3: 3 bytes at 3g).
__device__ __forceinline__ void store_group(uint8_t *row, int g, int bits, const int (&c)[8]) {
    if (bits == 4) {
        *reinterpret_cast<uint32_t *>(row + 4 * g) = pack8_int4(c);
    } else {
        const uint32_t w = pack8_int3(c);
        uint8_t *p = row + 3 * g;
        p[0] = uint8_t(w);
        p[1] = uint8_t(w >> 8);
        p[2] = uint8_t(w >> 16);
    }
}

// ---------------------------------------------------------------------------
// Block reductions (deterministic: fixed tree, no atomics).  `red` must hold
// blockDim.x / 32 entries; all threads must call.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Maximum over the warp of a non-negative float in one integer reduction: the
// bit patterns of non-negative IEEE floats order like unsigned integers.
__device__ __forceinline__ float warp_max_nonneg(float v) {
    return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v)));
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ float block_max(float v, float *red) {
    v = warp_max(v);
    const int w = threadIdx.x / kWarp, l = threadIdx.x % kWarp;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = red[0];
    for (int i = 1; i < int(blockDim.x / kWarp); ++i) r = fmaxf(r, red[i]);
    return r;
}

__device__ __forceinline__ double block_sum(double v, double *red) {
    v = warp_sum(v);
    const int w = threadIdx.x / kWarp, l = threadIdx.x % kWarp;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = red[0];
    for (int i = 1; i < int(blockDim.x / kWarp); ++i) r += red[i];
    return r;
}

}  // namespace rsq
