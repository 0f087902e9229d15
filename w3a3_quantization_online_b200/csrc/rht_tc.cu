// rht_tc.cu -- randomised Hadamard transform of order 4096 or 8192 + per-token
// symmetric quantiser, bf16 input; the first stage of the transform runs on
// the tensor cores.
//
// Infra Quant II, QuaRot / Background: v = H diag(s) x / sqrt(d) with the
// Sylvester H of order d = 2^12 or 2^13; QuaRot / Method: per-token symmetric
// absmax quantisation.
//
// A token row is the R x 64 matrix U[a][b] = s_i x_i (i = 64 a + b, R = d/64).
// The Sylvester matrix factors as H_d = H_R (x) H_64, so the transform is
// W = H_R U H_64:
//  * Y = H_R U (along a) is one tcgen05 product per group of tokens, with
//    M = N = K = 128.  For d = 4096 (R = 64) four tokens go at once:
//        D[(p, a)][(q, b)] = sum_{(p', a')} diag(H_64, H_64)[(p, a)][(p', a')] B[(p', a')][(q, b)]
//    with B the four TMA-loaded token tiles (token p + 2 q).  For d = 8192
//    (R = 128) two tokens go at once: D[a][(q, b)] = sum_a' H_128[a][a'] B[a'][(q, b)]
//    (token q).  The products are +-1 x bf16, exact; accumulation is fp32 in TMEM.
//  * W = Y H_64 (along b): each thread reads one row a of one token (64
//    columns) from TMEM and finishes it with register butterflies (packed
//    f32x2), then owns the 64 contiguous outputs [64 a, 64 a + 64).
// The signs are applied to the tiles in shared memory (XOR of the bf16 sign
// bits) before the product.  The 1/sqrt(d) factor goes to the scale.
//
// Pipeline (one CTA per SM, 16 warps): token groups (4 or 2 tokens) stream
// into 5 tile stages (32 KB each) by TMA; two warp groups (8 warps each) take
// alternate groups, each with two of the four 128-column TMEM slots, so one
// group's product overlaps its own previous epilogue and the other warp group's
// work.  A stage is refilled, five groups ahead, by the warp group whose
// product read it, as soon as that product is done (no producer warp: with 16
// warps a thread may hold 128 registers).  The row maximum is combined only
// among the warps that hold the token.  Programmatic dependent launch: the
// Hadamard operand and the sign masks are built while the previous kernel of
// the stream may still run; x and the outputs only after it completes.  Waits
// are bounded (device status word).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kGroupWarps = 8;                // one consumer warp group
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kConsumerGroups = 2;
constexpr int kThreads = kConsumerGroups * kGroupThreads;  // 16 warps: 128 registers each
constexpr int kStageBytes = 32768;            // one token group (4 x 8 KB or 2 x 16 KB)
constexpr int kStages = 5;
constexpr int kSlots = 4;                     // TMEM slots of 128 columns (two per warp group)

// Shape constants for token rows of d = 64 * ROWS elements.
template <int ROWS>
struct Shape {
    static constexpr int kD = 64 * ROWS;
    static constexpr int kTileBytes = ROWS * 128;             // one token: ROWS rows x 128 B (bf16)
    static constexpr int kTok = kStageBytes / kTileBytes;     // tokens per group: 4 or 2
    static constexpr int kQuadsPerToken = ROWS / 32;          // TMEM lane quadrants holding one token
    static constexpr int kOffA = 0;                           // H (block-diagonal for ROWS = 64), 2 x 16 KB
    static constexpr int kOffMask = kOffA + 2 * 16384;        // sign masks, laid out like a token tile
    static constexpr int kOffStage = kOffMask + kTileBytes;
    static constexpr int kOffRed = kOffStage + kStages * kStageBytes;  // [warp group][token][quadrant]
    static constexpr int kOffBar = kOffRed + kConsumerGroups * 8 * 4;
    static constexpr int kOffTmem = kOffBar + (kStages + kSlots) * 8;  // full[], mma[]
    static constexpr int kBytes = kOffTmem + 16;
    static constexpr int kSmem = kBytes + 1024;
    static_assert(kTok * kQuadsPerToken == 8, "reduction slots");
};

__device__ __forceinline__ uint32_t tile_off(int a, int chunk) {  // SWIZZLE_128B token tile
    return uint32_t(a * 128 + ((chunk ^ (a & 7)) << 4));
}

// In-place 64-point Sylvester transform of v[0..63], all stages but the last.
// Adjacent elements form the packed pairs (v[2j], v[2j+1]) -- the register
// pairs the TMEM load delivers -- so the stages for index bits 1..5 are packed
// two-wide butterflies between pairs; the stage for bit 0 works inside each
// pair (fwht64_last_absmax).
__device__ __forceinline__ void fwht64_outer(float (&v)[64]) {
#pragma unroll
    for (int hv = 1; hv < 32; hv <<= 1) {  // pair stride: element stride 2 hv
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if ((j & hv) == 0) {
                const float2 u = make_float2(v[2 * j], v[2 * j + 1]);
                const float2 w = make_float2(v[2 * (j + hv)], v[2 * (j + hv) + 1]);
                const float2 s = add2(u, w), d = sub2(u, w);
                v[2 * j] = s.x;
                v[2 * j + 1] = s.y;
                v[2 * (j + hv)] = d.x;
                v[2 * (j + hv) + 1] = d.y;
            }
        }
    }
}

// The last stage (inside each pair) and the largest magnitude of its outputs.
// max(|u + w|, |u - w|) = |u| + |w|, and rounding keeps the equality (the
// larger of the two rounded results is the rounded |u| + |w|), so the maximum
// is taken over the 32 pairs instead of the 64 outputs.
__device__ __forceinline__ float fwht64_last_absmax(float (&v)[64]) {
    float mx[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains of three-input maxima
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
        const float s0 = fabsf(v[2 * j]) + fabsf(v[2 * j + 1]);
        const float s1 = fabsf(v[2 * j + 2]) + fabsf(v[2 * j + 3]);
        mx[(j >> 1) & 3] = max3(mx[(j >> 1) & 3], s0, s1);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float u = v[2 * j], w = v[2 * j + 1];
        v[2 * j] = u + w;
        v[2 * j + 1] = u - w;
    }
    return max3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
}

// Codes of 64 values, 8 packed words (INT4) or 8 24-bit groups (INT3).  The
// row factor `pre` (1, or 2^64 for a tiny row) is always applied: one packed
// multiply per pair is cheaper than a per-element predicate.
template <int BITS, bool SCALED>
__device__ __forceinline__ void quant64s(const float (&v)[64], const RowQuant &rq, uint32_t (&w)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = v[8 * k + e];
        w[k] = pack8_fast<BITS>(f, rq.inv, rq.pre, SCALED);
    }
}

template <int ROWS, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
k_rht_tc(const __grid_constant__ CUtensorMap tm_x, const int8_t *__restrict__ signs,
         uint8_t *__restrict__ codes, float *__restrict__ scales, long long T, int *status) {
    using S = Shape<ROWS>;
    constexpr int kTok = S::kTok;
    constexpr int kTileBytes = S::kTileBytes;
    constexpr int kOffA = S::kOffA, kOffMask = S::kOffMask, kOffStage = S::kOffStage;
    constexpr int kOffRed = S::kOffRed, kOffBar = S::kOffBar, kOffTmem = S::kOffTmem;
    constexpr int qmax = (1 << (BITS - 1)) - 1;
    constexpr int row_bytes = S::kD * BITS / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_align1024(smem_raw);
    uint8_t *sa = base + kOffA;
    uint8_t *smask = base + kOffMask;
    uint8_t *sstage = base + kOffStage;
    const uint32_t bar_full = smem_u32(base + kOffBar);   // kStages: tile landed
    const uint32_t bar_mma = bar_full + 8 * kStages;      // kSlots: product done (its stage is free again)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffTmem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int err = 0;
    // programmatic dependent launch: the next kernel of the stream may start and
    // stage its constants now; it waits for this grid before it touches data
    asm volatile("griddepcontrol.launch_dependents;");

    // constants: A = diag(H_64, H_64) (ROWS = 64) or H_128 (ROWS = 128), with
    // H_n[a][a'] = (-1)^popcount(a & a'), bf16 +-1 (K-major, SWIZZLE_128B: slab kk
    // holds K columns 64 kk .. 64 kk + 63)
    for (int idx = tid; idx < 2 * 128 * 8; idx += kThreads) {
        const int kk = idx >> 10, m = (idx >> 3) & 127, ch = idx & 7;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t pair = 0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int k = 64 * kk + ch * 8 + 2 * e + u;
                uint32_t hv = 0;  // 0 outside the diagonal blocks of diag(H_64, H_64)
                if (ROWS == 128) hv = (__popc(m & k) & 1) ? 0xBF80u : 0x3F80u;
                else if ((m >> 6) == (k >> 6)) hv = (__popc((m & 63) & (k & 63)) & 1) ? 0xBF80u : 0x3F80u;
                pair |= hv << (16 * u);
            }
            w[e] = pair;
        }
        *reinterpret_cast<uint4 *>(sa + kk * 16384 + tile_off(m, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    // sign masks: bit 15 / 31 of the word for (a, b-pair) flips elements 64a + 2j, 64a + 2j + 1
    for (int idx = tid; idx < ROWS * 32; idx += kThreads) {
        const int a = idx >> 5, j = idx & 31;
        const int i = 64 * a + 2 * j;
        const uint32_t mk = (signs[i] < 0 ? 0x8000u : 0u) | (signs[i + 1] < 0 ? 0x80000000u : 0u);
        *reinterpret_cast<uint32_t *>(smask + tile_off(a, j >> 2) + (j & 3) * 4) = mk;
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
    // H and the sign masks are built above while the previous kernel of the
    // stream may still run; x and every output only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const long long ngroups = (T + kTok - 1) / kTok;
    const long long g0 = blockIdx.x, gstep = gridDim.x;
    const int nmine = g0 < ngroups ? int((ngroups - 1 - g0) / gstep + 1) : 0;

    // group it goes to stage it % kStages; the first kStages are issued here, the
    // others by the epilogue of the group that last used the stage
    auto load_group = [&](int it) {
        const int s = it % kStages;
        if (err) return;  // no arming without the load that completes it
        mbar_expect_tx(bar_full + 8 * s, kStageBytes);
        tma_load_3d(smem_u32(sstage + s * kStageBytes), &tm_x, 0, 0, int((g0 + it * gstep) * kTok), bar_full + 8 * s);
    };
    if (tid == 0)
        for (int it = 0; it < kStages && it < nmine; ++it) load_group(it);
    __syncwarp();
    {
        // ------------------------------------------------ consumer warp groups
        const int wg = warp / kGroupWarps;              // takes local groups wg, wg + 2, ...
        const int gtid = tid - wg * kGroupThreads;      // thread within the warp group
        const int gw = warp - wg * kGroupWarps;
        const uint32_t named = 1 + wg;
        float *sred = reinterpret_cast<float *>(base + kOffRed) + wg * 8;
        const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
        // epilogue mapping: TMEM lane (p, a) = 64 p + a (ROWS = 64) or a (ROWS = 128),
        // column half q
        const int quad = gw & 3, q = gw >> 2;
        const int lrow = quad * 32 + lane;
        const int p = ROWS == 64 ? lrow >> 6 : 0, a = lrow & (ROWS - 1);
        const int tslot = ROWS == 64 ? p + 2 * q : q;  // token within the group
        constexpr int QPT = S::kQuadsPerToken;
        const uint32_t named_tok = 3 + 4 * wg + tslot;  // barrier of the QPT warps holding one token
        // sign masks of this thread's chunks (the same positions in every group)
        constexpr int kChunksPerThread = (kStageBytes / 16) / kGroupThreads;
        constexpr int kMasks = (kTileBytes / 16) / kGroupThreads;  // distinct positions: 2 or 4
        uint4 mk[kMasks];
#pragma unroll
        for (int k = 0; k < kMasks; ++k) mk[k] = reinterpret_cast<const uint4 *>(smask)[gtid + k * kGroupThreads];

        auto epilogue = [&](int it) {
            const int slot = it % kSlots;
            if (!mbar_wait(bar_mma + 8 * slot, uint32_t((it / kSlots) & 1), err != 0)) err |= kErrMbarTimeout;
            // the product has read stage it % kStages: refill it
            if (gtid == 0 && it + kStages < nmine) load_group(it + kStages);
            __syncwarp();
            tc_fence_after();
            float v[64];
            {
                uint32_t r0[32], r1[32];
                const uint32_t taddr = tmem + (uint32_t(quad * 32) << 16) + uint32_t(slot * 128 + q * 64);
                tmem_ld32(taddr, r0);
                tmem_ld32(taddr + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    v[k] = __uint_as_float(r0[k]);
                    v[k + 32] = __uint_as_float(r1[k]);
                }
            }
            fwht64_outer(v);  // along b; then the last stage, which also gives the row's largest magnitude
            const float wm = warp_max_nonneg(fwht64_last_absmax(v));
            // the ROWS rows of a token live in QPT quadrants of column half q
            if (lane == 0) sred[tslot * QPT + (quad & (QPT - 1))] = wm;
            named_sync(named_tok, 32 * QPT);  // only the warps that hold this token
            float amax = sred[tslot * QPT];
#pragma unroll
            for (int k = 1; k < QPT; ++k) amax = fmaxf(amax, sred[tslot * QPT + k]);
            const long long t = (g0 + (long long)it * gstep) * kTok + tslot;
            if (t < T) {
                const RowQuant rq = row_quant(amax, qmax);
                uint32_t w[8];
                if (rq.pre == 1.0f)  // the same for the whole warp (one token)
                    quant64s<BITS, false>(v, rq, w);
                else
                    quant64s<BITS, true>(v, rq, w);
                uint8_t *dst = codes + t * row_bytes + a * (8 * BITS);
                if (BITS == 4) {
                    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
                } else {  // 8 groups of 24 bits -> 6 words
                    uint32_t o[6];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        o[3 * h + 0] = w[4 * h] | (w[4 * h + 1] << 24);
                        o[3 * h + 1] = (w[4 * h + 1] >> 8) | (w[4 * h + 2] << 16);
                        o[3 * h + 2] = (w[4 * h + 2] >> 16) | (w[4 * h + 3] << 8);
                    }
#pragma unroll
                    for (int h = 0; h < 3; ++h) reinterpret_cast<uint2 *>(dst)[h] = make_uint2(o[2 * h], o[2 * h + 1]);
                }
                if (a == 0) scales[t] = amax > 0.f ? amax / (float(qmax) * sqrtf(float(S::kD))) : 0.f;
            }
            // no barrier here: the warp group's next epilogue follows its next
            // pre-product barrier, which orders these sred reads and TMEM loads
            // before any later write
            tc_fence_before();
        };

        int prev = -1;
        for (int it = wg; it < nmine; it += kConsumerGroups) {
            const int s = it % kStages, slot = it % kSlots;
            if (!mbar_wait(bar_full + 8 * s, uint32_t((it / kStages) & 1), err != 0)) err |= kErrMbarTimeout;
            // apply the random signs to the group's tiles (XOR of bf16 sign bits)
            uint8_t *st = sstage + s * kStageBytes;
#pragma unroll
            for (int k = 0; k < kChunksPerThread; ++k) {
                const int c = gtid + k * kGroupThreads;  // 16-byte chunk within the stage
                uint4 xv = reinterpret_cast<uint4 *>(st)[c];
                const uint4 mv = mk[k % kMasks];         // same position in the mask tile
                xv.x ^= mv.x;
                xv.y ^= mv.y;
                xv.z ^= mv.z;
                xv.w ^= mv.w;
                reinterpret_cast<uint4 *>(st)[c] = xv;
            }
            fence_proxy_async_cta();
            tc_fence_before();
            named_sync(named, kGroupThreads);
            if (gtid == 0) {
                tc_fence_after();
                // A: K-major, K-steps of 16 are 32 bytes apart within a slab, slabs 16 KB apart.
                // B: MN-major, K rows 128 B apart (16 per K-step: 2 KB), the two 64-column
                //    atoms (column halves q = 0, 1) 16 KB apart.
                const uint64_t ad0 = smem_desc_sw128(smem_u32(sa), 1024);
                const uint64_t bd0 = smem_desc_sw128_lbo(smem_u32(st), 16384, 1024);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t aoff = uint32_t((k >> 2) * 16384 + (k & 3) * 32) >> 4;
                    const uint32_t boff = uint32_t(k * 2048) >> 4;
                    if (!err) umma_f16(tmem + uint32_t(slot * 128), ad0 + aoff, bd0 + boff, idesc, k != 0);
                }
                if (!err) umma_commit(bar_mma + 8 * slot);
            }
            __syncwarp();  // the other lanes wait here, not in a poll that competes with lane 0
            if (prev >= 0) epilogue(prev);
            prev = it;
        }
        if (prev >= 0) epilogue(prev);
    }

    tc_fence_before();
    // after a failed wait no further asynchronous work was issued: let what was
    // already in flight land before TMEM is freed and the CTA exits
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

template <int ROWS, int BITS>
cudaError_t launch_shape(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                         cudaStream_t st) {
    using S = Shape<ROWS>;
    static bool configured[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = k_rht_tc<ROWS, BITS>;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    EncodeTiledFn enc = encode_fn();
    int *status = device_status_word();
    if (!enc || !status) return cudaErrorInvalidValue;
    CUtensorMap map;
    const cuuint64_t dims[3] = {64, cuuint64_t(ROWS), cuuint64_t(T)};
    const cuuint64_t strides[2] = {128, cuuint64_t(S::kD) * 2};
    const cuuint32_t box[3] = {64, cuuint32_t(ROWS), cuuint32_t(S::kTok)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const long long ngroups = (T + S::kTok - 1) / S::kTok;
    long long grid = num_sms();
    if (grid > ngroups) grid = ngroups;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, map, signs, codes, scales, T, status);
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

bool rht_tc_supports(int d, int m, int dtype, int bits, long long T) {
    return (d == 4096 || d == 8192) && m == 1 && dtype == 1 && (bits == 3 || bits == 4) && T >= 1 &&
           T <= 0x7FFFFFFFLL;
}

cudaError_t launch_rht_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T, int d,
                          int bits, cudaStream_t s) {
    if (d == 8192)
        return bits == 4 ? launch_shape<128, 4>(x, signs, codes, scales, T, s)
                         : launch_shape<128, 3>(x, signs, codes, scales, T, s);
    return bits == 4 ? launch_shape<64, 4>(x, signs, codes, scales, T, s)
                     : launch_shape<64, 3>(x, signs, codes, scales, T, s);
}

}  // namespace rsq
