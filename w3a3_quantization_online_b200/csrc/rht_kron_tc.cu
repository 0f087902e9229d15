// rht_kron_tc.cu -- randomised Hadamard transform of order d = 12288 =
// 1024 x 12 (H_1024 (x) H_12, H_12 the Paley type-I matrix) + per-token INT4
// quantiser, bf16 input, with the largest stage on the tensor cores: the
// down_proj input of a 12288-wide FFN.
//
// Infra Quant II, QuaRot / Method: for d = 2^n m the online Hadamard is
// H_{2^n} (x) H_m, a fast Walsh-Hadamard transform along the stride-m index and
// a dense H_m on each contiguous group of m, the random signs first; the
// per-token symmetric absmax quantiser; 1/sqrt(d) goes to the scale.
//
// With i = 12 a + b (a < 1024, b < 12) and a = 8 a1 + a0 (a1 < 128, a0 < 8),
// i = 96 a1 + n with n = 12 a0 + b < 96, and the Sylvester factor splits as
// H_1024 = H_128 (x) H_8 (along a1 and a0).  A token row is thus the 128 x 96
// matrix B[a1][n] = s_i x_i, contiguous in memory, and
//     D[a1'][n] = sum_a1 H_128[a1'][a1] B[a1][n]
// is one tcgen05 product (M = K = 128, N = 128 with the columns 96..127 zero):
// +-1 x bf16 products, exact, fp32 accumulation in TMEM.  The row arrives by
// two TMA boxes of 64 columns x 128 rows from a 3-D view (96, 128, T) of x; the
// second box is filled with zeros beyond column 96.  The epilogue thread of
// TMEM lane a1' holds D[a1'][0..95], i.e. all (a0, b) of one a1', and finishes
// in registers: H_8 along a0 and the dense H_12 along b (packed f32x2), then
// the row absmax (one warp reduction and an exchange among the four warps of
// the token) and the codes of its 96 outputs i = 96 a1' .. 96 a1' + 95, which
// are 48 contiguous bytes.  No shuffles and no transposes.
//
// Pipeline (one CTA per SM, 8 warps): token rows stream into 4 stages of 32 KB;
// two warp groups of four warps take alternate rows, each with two 128-column
// TMEM slots, so a group's product overlaps its own previous epilogue and the
// other group's work.  The signs are XORed into the staged row from a mask tile
// laid out like a stage.  A stage is refilled, four rows ahead, by the warp
// group whose product read it.  Programmatic dependent launch: the Hadamard
// operand and the masks are built while the previous kernel of the stream may
// still run.  Waits are bounded (device status word); after a failed wait no
// barrier is armed and no asynchronous work is issued.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kKD = 12288;
constexpr int kNCols = 96;                   // (a0, b) columns of one a1 row
constexpr int kGroupWarps = 4;               // one per TMEM lane quadrant: one token row per group
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kConsumerGroups = 2;
constexpr int kThreads = kConsumerGroups * kGroupThreads;  // 8 warps
constexpr int kHalfBytes = 128 * 128;        // 128 rows x 64 bf16 columns: one box
constexpr int kStageBytes = 2 * kHalfBytes;  // one token row (columns 96..127 zero)
constexpr int kStages = 4;
constexpr int kSlots = 4;                    // TMEM slots of 128 columns (two per warp group)
constexpr int kOffA = 0;                     // H_128, K-major, 2 x 16 KB
constexpr int kOffMask = kOffA + 2 * 16384;  // sign masks laid out like a stage (32 KB)
constexpr int kOffStage = kOffMask + kStageBytes;
constexpr int kOffRed = kOffStage + kStages * kStageBytes;  // [warp group][warp] row maxima
constexpr int kOffBar = kOffRed + kConsumerGroups * kGroupWarps * 4;
constexpr int kOffTmem = kOffBar + (kStages + kSlots) * 8;
constexpr int kBytes = kOffTmem + 16;
constexpr int kSmem = kBytes + 1024;
static_assert(kOffStage % 1024 == 0 && kOffMask % 1024 == 0, "swizzle atoms");
static_assert(kSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {  // SWIZZLE_128B, 128-byte rows
    return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Paley type-I Hadamard matrix of order 12: H = I + S, S = [[0, 1^T], [-1, J]],
// J[i][j] = chi(j - i) with chi the quadratic character mod 11 (nonzero squares
// 1, 3, 4, 5, 9).
__host__ __device__ constexpr int square_mod11(int q) { return q == 0 ? 1 : (q == 1 ? 3 : (q == 2 ? 4 : (q == 3 ? 5 : 9))); }
__host__ __device__ constexpr int paley12(int i, int j) {
    return i == j ? 1 : (i == 0 ? 1 : (j == 0 ? -1 : (((0x23A >> ((j - i + 11) % 11)) & 1) ? 1 : -1)));
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

// out = H_12 u on two groups at once (u[k] = (group 0, group 1) entries k).  With
// s = u_1 + ... + u_11 and P_i the sum of the u_j (1 <= j <= 11) with j - i a
// nonzero square mod 11, row i >= 1 of I + S gives
//     out_i = u_i - u_0 + (P_i - (s - u_i - P_i)) = 2 (u_i + P_i) - (u_0 + s)
// and row 0 (all ones) out_0 = u_0 + s.
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

// Low nibbles of 8 codes (the low bits of the rounded floats r[k]) -> one word,
// code k in nibble k.
__device__ __forceinline__ uint32_t nibbles8(const uint32_t (&r)[8]) {
    const uint32_t ev = prmt(prmt(r[0], r[2], 0x0040u), prmt(r[4], r[6], 0x0040u), 0x5410u);
    const uint32_t od = prmt(prmt(r[1], r[3], 0x0040u), prmt(r[5], r[7], 0x0040u), 0x5410u);
    return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
}

// Codes of the 96 values w[p][b] = (v[12 (2p) + b], v[12 (2p + 1) + b]) in output
// order n = 12 a0 + b: 12 words, words 3p .. 3p + 2 holding groups 2p and 2p + 1.
template <bool SCALED>
__device__ __forceinline__ void quant_pairs(const float2 (&w)[4][12], const RowQuant &rq, uint32_t (&out)[12]) {
    const float2 inv2 = make_float2(rq.inv, rq.inv), mag2 = make_float2(kRoundMagic, kRoundMagic);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        uint32_t e[12], o[12];  // rounded codes of group 2p (even) and 2p + 1 (odd)
#pragma unroll
        for (int b = 0; b < 12; ++b) {
            float2 t = w[p][b];
            if (SCALED) t = mul2(t, make_float2(rq.pre, rq.pre));
            const float2 q = fma2(t, inv2, mag2);  // |v| <= amax: no clamp needed
            e[b] = __float_as_uint(q.x);
            o[b] = __float_as_uint(q.y);
        }
        const uint32_t r0[8] = {e[0], e[1], e[2], e[3], e[4], e[5], e[6], e[7]};
        const uint32_t r1[8] = {e[8], e[9], e[10], e[11], o[0], o[1], o[2], o[3]};
        const uint32_t r2[8] = {o[4], o[5], o[6], o[7], o[8], o[9], o[10], o[11]};
        out[3 * p] = nibbles8(r0);
        out[3 * p + 1] = nibbles8(r1);
        out[3 * p + 2] = nibbles8(r2);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
k_rht_kron_tc(const __grid_constant__ CUtensorMap tm_x, const int8_t *__restrict__ signs,
              uint8_t *__restrict__ codes, float *__restrict__ scales, long long T, int *status) {
    constexpr int qmax = 7;
    constexpr int row_bytes = kKD / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_align1024(smem_raw);
    uint8_t *sa = base + kOffA;
    uint8_t *smask = base + kOffMask;
    uint8_t *sstage = base + kOffStage;
    const uint32_t bar_full = smem_u32(base + kOffBar);  // kStages: row landed
    const uint32_t bar_mma = bar_full + 8 * kStages;     // kSlots: product done (its stage is free again)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffTmem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int err = 0;
    asm volatile("griddepcontrol.launch_dependents;");

    // A = H_128[m][k] = (-1)^popcount(m & k), bf16 +-1, K-major, SWIZZLE_128B:
    // slab kk holds K columns 64 kk .. 64 kk + 63
    for (int idx = tid; idx < 2 * 128 * 8; idx += kThreads) {
        const int kk = idx >> 10, m = (idx >> 3) & 127, ch = idx & 7;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t pair = 0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int k = 64 * kk + ch * 8 + 2 * e + u;
                pair |= ((__popc(m & k) & 1) ? 0xBF80u : 0x3F80u) << (16 * u);
            }
            w[e] = pair;
        }
        *reinterpret_cast<uint4 *>(sa + kk * 16384 + tile_off(m, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    // sign masks laid out like a staged row: half q, row a1, physical chunk p holds
    // columns n = 64 q + 8 (p ^ (a1 & 7)) .. +8 of row a1 (i = 96 a1 + n; none past 96)
    for (int idx = tid; idx < 2 * 128 * 8; idx += kThreads) {
        const int q = idx >> 10, a1 = (idx >> 3) & 127, pch = idx & 7;
        const int n0 = 64 * q + 8 * (pch ^ (a1 & 7));
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = n0 + 2 * e;
            uint32_t mk = 0;
            if (n < kNCols) mk |= signs[kNCols * a1 + n] < 0 ? 0x8000u : 0u;
            if (n + 1 < kNCols) mk |= signs[kNCols * a1 + n + 1] < 0 ? 0x80000000u : 0u;
            w[e] = mk;
        }
        *reinterpret_cast<uint4 *>(smask + q * kHalfBytes + a1 * 128 + pch * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(bar_full + 8 * s, 1);
        for (int s = 0; s < kSlots; ++s) mbar_init(bar_mma + 8 * s, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kSlots * 128);
        tmem_relinquish();
    }
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const long long r0 = blockIdx.x, rstep = gridDim.x;
    const int nmine = r0 < T ? int((T - 1 - r0) / rstep + 1) : 0;

    // row it goes to stage it % kStages as two 64-column boxes 16 KB apart
    auto load_row = [&](int it) {
        const int s = it % kStages;
        if (err) return;  // no arming without the loads that complete it
        const int t = int(r0 + (long long)it * rstep);
        mbar_expect_tx(bar_full + 8 * s, kStageBytes);
        tma_load_3d(smem_u32(sstage + s * kStageBytes), &tm_x, 0, 0, t, bar_full + 8 * s);
        tma_load_3d(smem_u32(sstage + s * kStageBytes + kHalfBytes), &tm_x, 64, 0, t, bar_full + 8 * s);
    };
    if (tid == 0)
        for (int it = 0; it < kStages && it < nmine; ++it) load_row(it);
    __syncwarp();
    {
        const int wg = warp / kGroupWarps;  // takes local rows wg, wg + 2, ...
        const int gtid = tid - wg * kGroupThreads;
        const int gw = warp - wg * kGroupWarps;  // == TMEM lane quadrant
        const int a1 = 32 * gw + lane;           // this thread's row of D
        const uint32_t named = 1 + wg;
        float *sred = reinterpret_cast<float *>(base + kOffRed) + wg * kGroupWarps;
        const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);

        auto epilogue = [&](int it) {
            const int slot = it % kSlots;
            if (!mbar_wait(bar_mma + 8 * slot, uint32_t((it / kSlots) & 1), err != 0)) err |= kErrMbarTimeout;
            // the product has read stage it % kStages: refill it
            if (gtid == 0 && it + kStages < nmine) load_row(it + kStages);
            __syncwarp();
            tc_fence_after();
            // w[p][b] = (D[a1][12 (2p) + b], D[a1][12 (2p + 1) + b]): one pairing of the
            // values for every step, so that the packed operations need no moves
            float2 w[4][12];
            {
                uint32_t r[32];
                const uint32_t taddr = tmem + (uint32_t(gw * 32) << 16) + uint32_t(slot * 128);
#pragma unroll
                for (int h = 0; h < 3; ++h) {
                    tmem_ld32(taddr + 32 * h, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int n = 32 * h + k, a0 = n / 12, b = n % 12;
                        if (a0 & 1) w[a0 >> 1][b].y = __uint_as_float(r[k]);
                        else w[a0 >> 1][b].x = __uint_as_float(r[k]);
                    }
                }
            }
            // H_8 along a0: bit 0 inside each pair, bits 1 and 2 between pairs
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int b = 0; b < 12; ++b) w[p][b] = make_float2(w[p][b].x + w[p][b].y, w[p][b].x - w[p][b].y);
#pragma unroll
            for (int s = 1; s < 4; s <<= 1)
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    if (!(p & s))
#pragma unroll
                        for (int b = 0; b < 12; ++b) {
                            const float2 u = w[p][b], x = w[p | s][b];
                            w[p][b] = add2(u, x);
                            w[p | s][b] = sub2(u, x);
                        }
            // dense H_12 along b on groups 2p and 2p + 1 at once
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                float2 o[12];
                h12_pair(w[p], o);
#pragma unroll
                for (int k = 0; k < 12; ++k) w[p][k] = o[k];
            }
            float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int b = 0; b < 12; ++b) mx[b & 3] = max3(mx[b & 3], fabsf(w[p][b].x), fabsf(w[p][b].y));
            const float wm = warp_max_nonneg(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
            if (lane == 0) sred[gw] = wm;
            named_sync(named, kGroupThreads);  // the four warps of this row
            const float amax = fmaxf(fmaxf(sred[0], sred[1]), fmaxf(sred[2], sred[3]));
            const long long t = r0 + (long long)it * rstep;
            const RowQuant rq = row_quant(amax, qmax);
            uint32_t wd[12];
            if (rq.pre == 1.0f)  // the same for the whole row
                quant_pairs<false>(w, rq, wd);
            else
                quant_pairs<true>(w, rq, wd);
            uint4 *dst = reinterpret_cast<uint4 *>(codes + t * row_bytes + 48 * a1);
#pragma unroll
            for (int k = 0; k < 3; ++k) dst[k] = make_uint4(wd[4 * k], wd[4 * k + 1], wd[4 * k + 2], wd[4 * k + 3]);
            if (gtid == 0) scales[t] = amax > 0.f ? amax / (float(qmax) * sqrtf(float(kKD))) : 0.f;
            // no barrier here: the group's next epilogue follows its next pre-product
            // barrier, which orders these sred reads and TMEM loads before any later write
            tc_fence_before();
        };

        int prev = -1;
        for (int it = wg; it < nmine; it += kConsumerGroups) {
            const int s = it % kStages, slot = it % kSlots;
            if (!mbar_wait(bar_full + 8 * s, uint32_t((it / kStages) & 1), err != 0)) err |= kErrMbarTimeout;
            // the random signs: XOR of the bf16 sign bits, chunk by chunk as laid out
            uint4 *st = reinterpret_cast<uint4 *>(sstage + s * kStageBytes);
            const uint4 *mk = reinterpret_cast<const uint4 *>(smask);
#pragma unroll 4
            for (int k = 0; k < kStageBytes / 16 / kGroupThreads; ++k) {
                const int c = gtid + k * kGroupThreads;
                uint4 xv = st[c];
                const uint4 mv = mk[c];
                xv.x ^= mv.x;
                xv.y ^= mv.y;
                xv.z ^= mv.z;
                xv.w ^= mv.w;
                st[c] = xv;
            }
            fence_proxy_async_cta();
            tc_fence_before();
            named_sync(named, kGroupThreads);
            if (gtid == 0) {
                tc_fence_after();
                // A: K-major, K-steps of 16 are 32 bytes apart within a slab, slabs 16 KB apart.
                // B: MN-major, K rows 128 B apart (16 per K-step: 2 KB), the two 64-column
                //    boxes 16 KB apart.
                const uint64_t ad0 = smem_desc_sw128(smem_u32(sa), 1024);
                const uint64_t bd0 = smem_desc_sw128_lbo(smem_u32(sstage + s * kStageBytes), kHalfBytes, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t aoff = uint32_t((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                    const uint32_t boff = uint32_t(k * 2048) >> 4;
                    if (!err) umma_f16(tmem + uint32_t(slot * 128), ad0 + aoff, bd0 + boff, idesc, k != 0);
                }
                if (!err) umma_commit(bar_mma + 8 * slot);
            }
            __syncwarp();
            if (prev >= 0) epilogue(prev);
            prev = it;
        }
        if (prev >= 0) epilogue(prev);
    }

    tc_fence_before();
    if (__syncthreads_or(err)) drain_delay();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kSlots * 128);
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(status, err);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

}  // namespace

bool rht_kron_tc_supports(int d, int m, int dtype, int bits, long long T) {
    return d == kKD && m == 12 && dtype == 1 && bits == 4 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_rht_kron_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                               cudaStream_t s) {
    static bool configured[64];
    static EncodeTiledFn enc = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(k_rht_kron_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    if (!enc) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return cudaErrorInvalidValue;
        enc = reinterpret_cast<EncodeTiledFn>(p);
    }
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidValue;
    // x as (96, 128, T): column n of row a1 of token t is x_t[96 a1 + n]
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(kNCols), 128, cuuint64_t(T)};
    const cuuint64_t strides[2] = {cuuint64_t(kNCols) * 2, cuuint64_t(kKD) * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    long long grid = num_sms();
    if (grid > T) grid = T;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_rht_kron_tc, map, signs, codes, scales, T, status);
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace rsq
