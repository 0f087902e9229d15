// rht_kron.cu -- the gated down_proj input of a 12288-wide FFN, g = SiLU(a) * b
// in fp32, through the randomised Hadamard transform of order d = 12288 =
// 1024 x 12 (H_1024 (x) H_12, H_12 the Paley type-I matrix, q = 11) and the
// per-token INT4 quantiser, bf16 inputs.  (Without the gate the tensor-core
// kernel of rht_kron_tc.cu serves this transform.)
//
// Infra Quant II, QuaRot / Method: for d = 2^n m the online Hadamard is
// H_{2^n} (x) H_m, applied as a fast Walsh-Hadamard transform along the stride-m
// index and a dense H_m on each contiguous group of m; the random signs first;
// the online Hadamard sits on the down_proj input.  QuaRot / Method:
// per-token symmetric absmax quantisation; 1/sqrt(d) goes to the scale.
//
// One CTA per token row at a time (two CTAs per SM), 256 threads; the next rows
// of a and b are staged in shared memory by bulk copies while the current one
// is transformed (bounded wait, device status word).  With i = 12 a + b
// (a < 1024, b < 12), thread t first owns the four groups a = 4t..4t+3 (48
// contiguous values):
//   1. load a and b, the gate SiLU(a) * b in fp32 (never rounded to bf16), the
//      signs on the fp32 sign bit (48 sign bits per thread), dense H_12 on each
//      group in registers (packed f32x2 over pairs of groups);
//   2. FWHT along a: bits 0-1 in the thread, bits 2-6 (the lane) by warp
//      shuffles;
//   3. one transpose through shared memory (blocks padded to 52 floats against
//      bank conflicts) so that thread (a0, h) owns a = a0 + 128 k (k < 8) and
//      b = 6h..6h+5; FWHT bits 7-9 in the thread;
//   4. block absmax, codes of 6 consecutive columns per (thread, k) = 3 bytes.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kKThreads = 256;
constexpr int kKd = 12288;
constexpr int kKBlk = 52;  // floats per thread block of 48 in the transpose buffer

// Paley type-I Hadamard matrix of order 12: H = I + S, S = [[0, 1^T], [-1, J]],
// J[i][j] = chi(j - i) with chi the quadratic character mod 11 (nonzero squares:
// 1, 3, 4, 5, 9 -> bit mask 0x23A).
__host__ __device__ constexpr int paley12(int i, int j) {
    return i == j ? 1 : (i == 0 ? 1 : (j == 0 ? -1 : (((0x23A >> ((j - i + 11) % 11)) & 1) ? 1 : -1)));
}

// The residue neighbours used below are exactly the +1 entries of the Paley
// rows 1..11 off the diagonal and column 0: checked at compile time.
__host__ __device__ constexpr int square_mod11(int q) {  // the nonzero squares mod 11: 1, 3, 4, 5, 9
    return q == 0 ? 1 : (q == 1 ? 3 : (q == 2 ? 4 : (q == 3 ? 5 : 9)));
}
constexpr bool paley_rows_match_residues() {
    for (int i = 1; i < 12; ++i) {
        int plus = 0;
        for (int j = 1; j < 12; ++j)
            if (j != i && paley12(i, j) == 1) ++plus;
        if (plus != 5) return false;
        for (int q = 0; q < 5; ++q)
            if (paley12(i, (i - 1 + square_mod11(q)) % 11 + 1) != 1) return false;
        if (paley12(i, 0) != -1 || paley12(0, i) != 1 || paley12(i, i) != 1) return false;
    }
    return paley12(0, 0) == 1;
}
static_assert(paley_rows_match_residues(), "Paley H_12 structure");

// out = H_12 u on two groups at once (u[k] = (group 0, group 1) entries k).
// With s = u_1 + ... + u_11 and P_i = sum of u_j over the j (1..11) with
// chi(j - i) = +1 (j - i a nonzero square mod 11), row i >= 1 of I + S gives
//     out_i = u_i - u_0 + (P_i - (s - u_i - P_i)) = 2 (u_i + P_i) - (u_0 + s),
// and row 0 (all ones) gives out_0 = u_0 + s: 6 packed operations per output
// instead of 11.
__device__ __forceinline__ void h12_pair(const float2 (&u)[12], float2 (&out)[12]) {
    float2 s = u[1];
#pragma unroll
    for (int k = 2; k < 12; ++k) s = add2(s, u[k]);
    const float2 c = add2(u[0], s);
    out[0] = c;
#pragma unroll
    for (int i = 1; i < 12; ++i) {
        float2 acc = u[i];
#pragma unroll
        for (int q = 0; q < 5; ++q) acc = add2(acc, u[(i - 1 + square_mod11(q)) % 11 + 1]);
        out[i] = fma2(acc, make_float2(2.f, 2.f), make_float2(-c.x, -c.y));
    }
}

template <int BITS>
__global__ void __launch_bounds__(kKThreads, 2)
k_rht_kron_gate(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ xb,
           const int8_t *__restrict__ signs, uint8_t *__restrict__ codes,
           float *__restrict__ scales, long long T, int *status) {
    static_assert(BITS == 4, "6 codes of 4 bits make 3 whole bytes");
    extern __shared__ float4 km4[];
    float *buf = reinterpret_cast<float *>(km4);                    // 256 x 52 floats
    uint64_t *sbits = reinterpret_cast<uint64_t *>(buf + kKThreads * kKBlk);  // 48 sign bits per thread
    uint4 *srow = reinterpret_cast<uint4 *>(sbits + kKThreads);     // the row of a being processed (bf16)
    uint4 *srow_b = srow + kKd / 8;                                 // the row of b
    __shared__ float red[kKThreads / 32];
    __shared__ __align__(8) uint64_t bar_row;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t bar = smem_u32(&bar_row);
    int err = 0;
    constexpr int qmax = 7;
    constexpr int row_bytes = kKd / 2;

    {
        uint64_t w = 0;  // bit e: sign of element 48 tid + e
        for (int e = 0; e < 48; ++e) w |= uint64_t(signs[48 * tid + e] < 0) << e;
        sbits[tid] = w;
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        if (blockIdx.x < T) {  // the first row (the next ones are staged while the previous is transformed)
            mbar_expect_tx(bar, 2 * kKd * 2);
            bulk_load_1d(smem_u32(srow), x + (long long)blockIdx.x * kKd, kKd * 2, bar);
            bulk_load_1d(smem_u32(srow_b), xb + (long long)blockIdx.x * kKd, kKd * 2, bar);
        }
    }
    __syncthreads();

    const float2 one2 = make_float2(1.f, 1.f), mone2 = make_float2(-1.f, -1.f);
    const int a0 = tid & 127, hb = tid >> 7;  // owner after the transpose

    int it = 0;
    for (long long t = blockIdx.x; t < T; t += gridDim.x, ++it) {
        // ---- 1. 48 values (groups a = 4 tid + g) from the staged row, signs, H_12
        if (!mbar_wait(bar, uint32_t(it) & 1u, err != 0)) err |= kErrMbarTimeout;
        float2 p[2][12];  // p[h][k] = (group 2h, group 2h+1) entry k
        {
            const uint4 *src = srow + 6 * tid, *srcb = srow_b + 6 * tid;
            const uint64_t sb = sbits[tid];
#pragma unroll
            for (int c = 0; c < 6; ++c) {
                const uint4 u = src[c], ub = srcb[c];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int e = 8 * c + q, g = e / 12, k = e % 12;
                    const float fa = __uint_as_float(q & 1 ? (w[q >> 1] & 0xFFFF0000u) : (w[q >> 1] << 16));
                    const float fb = __uint_as_float(q & 1 ? (wb[q >> 1] & 0xFFFF0000u) : (wb[q >> 1] << 16));
                    const float f = __uint_as_float(__float_as_uint(silu_gate(fa, fb)) ^
                                                    (uint32_t((sb >> e) & 1u) << 31));
                    if (g & 1) p[g >> 1][k].y = f;
                    else p[g >> 1][k].x = f;
                }
            }
            fence_proxy_async_cta();  // these reads before the next row's bulk copies
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 o[12];
            h12_pair(p[h], o);
#pragma unroll
            for (int k = 0; k < 12; ++k) p[h][k] = o[k];
        }
        // ---- 2. FWHT along a: bit 1 (pairs of groups), bit 0 (inside a pair)
#pragma unroll
        for (int k = 0; k < 12; ++k) {
            const float2 s = add2(p[0][k], p[1][k]), d = sub2(p[0][k], p[1][k]);
            p[0][k] = s;
            p[1][k] = d;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < 12; ++k) {
                const float u = p[h][k].x, w = p[h][k].y;
                p[h][k] = make_float2(u + w, u - w);
            }
        // bits 2-6: the lane; the upper partner forms (lower - upper) = partner - own
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const float2 sg = (lane & m) ? mone2 : one2;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int k = 0; k < 12; ++k) {
                    const float2 q = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p[h][k].x, m),
                                                 __shfl_xor_sync(0xFFFFFFFFu, p[h][k].y, m));
                    p[h][k] = fma2(p[h][k], sg, q);
                }
        }
        // ---- 3. transpose: element (g, k) of thread tid at buf[tid * 52 + 12 g + k]
        {
            float *dst = buf + tid * kKBlk;
#pragma unroll
            for (int j = 0; j < 12; ++j) {
                float f[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int e = 4 * j + q, g = e / 12, k = e % 12;
                    f[q] = (g & 1) ? p[g >> 1][k].y : p[g >> 1][k].x;
                }
                *reinterpret_cast<float4 *>(dst + 4 * j) = make_float4(f[0], f[1], f[2], f[3]);
            }
        }
        __syncthreads();  // the staged row is consumed: bring in the next one
        if (tid == 0 && t + gridDim.x < T && !err) {  // no arming without the loads that complete it
            mbar_expect_tx(bar, 2 * kKd * 2);
            bulk_load_1d(smem_u32(srow), x + (t + gridDim.x) * kKd, kKd * 2, bar);
            bulk_load_1d(smem_u32(srow_b), xb + (t + gridDim.x) * kKd, kKd * 2, bar);
        }
        // thread (a0, hb) now takes a = a0 + 128 k (k < 8), b = 6 hb .. 6 hb + 5
        float2 r[8][3];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int a = a0 + 128 * k;
            const float *srcp = buf + (a >> 2) * kKBlk + 12 * (a & 3) + 6 * hb;
#pragma unroll
            for (int j = 0; j < 3; ++j) r[k][j] = *reinterpret_cast<const float2 *>(srcp + 2 * j);
        }
        // FWHT bits 7-9 of a: k bits 0-2
#pragma unroll
        for (int s = 1; s < 8; s <<= 1)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (!(k & s))
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        const float2 u = r[k][j], w = r[k | s][j];
                        r[k][j] = add2(u, w);
                        r[k | s][j] = sub2(u, w);
                    }
        // ---- 4. absmax over the row, codes, scale
        float m0 = 0.f, m1 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                if (j & 1) m1 = max3(m1, fabsf(r[k][j].x), fabsf(r[k][j].y));
                else m0 = max3(m0, fabsf(r[k][j].x), fabsf(r[k][j].y));
            }
        const float wm = warp_max(fmaxf(m0, m1));
        if (lane == 0) red[warp] = wm;
        __syncthreads();  // also: every thread has read the transpose buffer
        float amax = red[0];
#pragma unroll
        for (int w = 1; w < kKThreads / 32; ++w) amax = fmaxf(amax, red[w]);
        const RowQuant rq = row_quant(amax, qmax);
        const float2 inv2 = make_float2(rq.inv, rq.inv), pre2 = make_float2(rq.pre, rq.pre);
        const float2 mag2 = make_float2(kRoundMagic, kRoundMagic);
        uint8_t *crow = codes + t * row_bytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            uint32_t c[6];
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                // |v| <= amax: |v qmax / amax| <= qmax, no clamp needed
                const float2 q = fma2(mul2(r[k][j], pre2), inv2, mag2);
                c[2 * j] = __float_as_uint(q.x);
                c[2 * j + 1] = __float_as_uint(q.y);
            }
            uint8_t *dst = crow + 6 * (a0 + 128 * k) + 3 * hb;  // codes 12 a + 6 hb .. + 5
            dst[0] = uint8_t((c[0] & 0xFu) | ((c[1] & 0xFu) << 4));
            dst[1] = uint8_t((c[2] & 0xFu) | ((c[3] & 0xFu) << 4));
            dst[2] = uint8_t((c[4] & 0xFu) | ((c[5] & 0xFu) << 4));
        }
        if (tid == 0) scales[t] = amax > 0.f ? amax / (float(qmax) * sqrtf(float(kKd))) : 0.f;
        __syncthreads();  // red[] and the transpose buffer are reused by the next row
    }
    if (__syncthreads_or(err)) drain_delay();  // a staged copy still in flight lands before the CTA exits
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(status, err);
}

}  // namespace

bool rht_kron_gate_supports(int d, int m, int dtype, int bits, long long T) {
    return d == kKd && m == 12 && dtype == 1 && bits == 4 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_rht_kron_gate(const void *a, const void *b, const int8_t *signs, uint8_t *codes, float *scales,
                                 long long T, cudaStream_t s) {
    static bool configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // transpose buffer; 48 sign bits per thread; the staged rows of a and b
    const size_t smem = size_t(kKThreads) * kKBlk * 4 + size_t(kKThreads) * 8 + size_t(kKd) * 2 * 2;
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidValue;
    auto kern = k_rht_kron_gate<4>;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const long long cap = (long long)num_sms() * 2;
    const int grid = int(T < cap ? T : cap);
    kern<<<grid, kKThreads, smem, s>>>(static_cast<const __nv_bfloat16 *>(a), static_cast<const __nv_bfloat16 *>(b),
                                       signs, codes, scales, T, status);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace rsq
