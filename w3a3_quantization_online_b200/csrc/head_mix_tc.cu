// head_mix_tc.cu -- head mixing of the attention output (the out_proj input)
// on the tensor cores, then per-token symmetric quantiser: bf16 input, 32 heads
// of 128.
//
// Infra Quant II, QuaRot / Method: the attention output is rotated across the
// heads, v = (H_{n_h} (x) I_{d_h}) diag(s) x / sqrt(n_h) (the n_h-point
// Sylvester transform along the head index at stride d_h), and quantised per
// token with the symmetric absmax scale (SpinQuant / Motivation:
// alpha = max|X| / (2^(N-1) - 1)).
//
// A token row is the 32 x 128 matrix X[h][j] = s_i x_i (i = 128 h + j), so the
// transform of four tokens at once is one tcgen05 product with M = N = K = 128:
//     D[(t, h')][j] = sum_{(t', h)} diag(H_32, H_32, H_32, H_32)[(t, h')][(t', h)] B[(t', h)][j]
// with B the four tokens' rows stacked (row (t, h) = x_t[128 h .. 128 h + 127]),
// which is exactly their layout in memory: one 2-D TMA box of 128 rows per
// 64-column half.  The products are +-1 x bf16, exact; the accumulation is
// fp32 in TMEM.  The 1/sqrt(32) factor goes to the scale.
//
// Pipeline (one CTA per SM, 16 warps): token groups stream into 5 stages of
// 32 KB; two warp groups take alternate groups, each with two of the four
// 128-column TMEM slots, so one group's product overlaps its own previous
// epilogue and the other group's work.  The signs are applied to the tile in
// shared memory (XOR of the bf16 sign bits; skipped without signs).  Epilogue:
// TMEM lane quadrant t holds token t (lane = head h'), the two column halves go
// to two warps, so a token's absmax is one warp reduction and one exchange
// between two warps; each thread then writes the codes of its 64 outputs
// [128 h' + 64 q, +64).  A stage is refilled, five groups ahead, by the warp
// group whose product read it.  Programmatic dependent launch: the Hadamard
// operand and the sign masks are built while the previous kernel of the stream
// may still run.  Waits are bounded (device status word); after a failed wait
// no barrier is armed and no asynchronous work is issued.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kNH = 32;                       // heads
constexpr int kDH = 128;                      // head width
constexpr int kD = kNH * kDH;                 // 4096
constexpr int kTok = 128 / kNH;               // tokens per group (product M = 128)
constexpr int kGroupWarps = 8;
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kConsumerGroups = 2;
constexpr int kThreads = kConsumerGroups * kGroupThreads;  // 16 warps
constexpr int kHalfBytes = 128 * 128;         // 128 rows x 64 bf16: one column half of a group
constexpr int kStageBytes = 2 * kHalfBytes;   // 32 KB: four tokens
constexpr int kStages = 5;
constexpr int kSlots = 4;                     // TMEM slots of 128 columns (two per warp group)
constexpr int kOffA = 0;                      // diag(H_32 x 4), K-major, 2 x 16 KB
constexpr int kOffMask = kOffA + 2 * 16384;   // sign masks: [half][head][128 B], swizzled like a tile
constexpr int kOffStage = kOffMask + 2 * 32 * 128;
constexpr int kOffRed = kOffStage + kStages * kStageBytes;  // [warp group][token][half] row maxima
constexpr int kOffBar = kOffRed + kConsumerGroups * kTok * 2 * 4;
constexpr int kOffTmem = kOffBar + (kStages + kSlots) * 8;
constexpr int kBytes = kOffTmem + 16;
constexpr int kSmem = kBytes + 1024;
static_assert(kOffStage % 1024 == 0, "swizzle atoms");
static_assert(kSmem <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {  // SWIZZLE_128B, 128-byte rows
    return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Codes of 64 values: 8 packed words (INT4) or 8 groups of 24 bits (INT3).
template <int BITS, bool SCALED>
__device__ __forceinline__ void quant64(const float (&v)[64], const RowQuant &rq, uint32_t (&w)[8]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = v[8 * k + e];
        w[k] = pack8_fast<BITS>(f, rq.inv, rq.pre, SCALED);
    }
}

template <int BITS, bool SIGNS>
__global__ void __launch_bounds__(kThreads, 1)
k_head_mix_tc(const __grid_constant__ CUtensorMap tm_x, const int8_t *__restrict__ signs,
              uint8_t *__restrict__ codes, float *__restrict__ scales, long long T, int *status) {
    constexpr int qmax = (1 << (BITS - 1)) - 1;
    constexpr int row_bytes = kD * BITS / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_align1024(smem_raw);
    uint8_t *sa = base + kOffA;
    uint8_t *smask = base + kOffMask;
    uint8_t *sstage = base + kOffStage;
    const uint32_t bar_full = smem_u32(base + kOffBar);  // kStages: group landed
    const uint32_t bar_mma = bar_full + 8 * kStages;     // kSlots: product done (its stage is free again)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffTmem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int err = 0;
    asm volatile("griddepcontrol.launch_dependents;");

    // A = diag(H_32, H_32, H_32, H_32), H_32[h'][h] = (-1)^popcount(h' & h), bf16 +-1,
    // K-major, SWIZZLE_128B: slab kk holds K columns 64 kk .. 64 kk + 63
    for (int idx = tid; idx < 2 * 128 * 8; idx += kThreads) {
        const int kk = idx >> 10, m = (idx >> 3) & 127, ch = idx & 7;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t pair = 0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int k = 64 * kk + ch * 8 + 2 * e + u;
                uint32_t hv = 0;  // 0 outside the diagonal blocks
                if ((m >> 5) == (k >> 5)) hv = (__popc((m & 31) & (k & 31)) & 1) ? 0xBF80u : 0x3F80u;
                pair |= hv << (16 * u);
            }
            w[e] = pair;
        }
        *reinterpret_cast<uint4 *>(sa + kk * 16384 + tile_off(m, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    // sign masks: for column half q and head h, physical chunk p of the swizzled
    // row holds columns 64 q + 8 (p ^ (h & 7)) .. +8, one bf16 sign bit each
    if (SIGNS) {
        for (int idx = tid; idx < 2 * 32 * 8; idx += kThreads) {
            const int q = idx >> 8, h = (idx >> 3) & 31, pch = idx & 7;
            const int j0 = 64 * q + 8 * (pch ^ (h & 7));
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = kDH * h + j0 + 2 * e;
                w[e] = (signs[i] < 0 ? 0x8000u : 0u) | (signs[i + 1] < 0 ? 0x80000000u : 0u);
            }
            *reinterpret_cast<uint4 *>(smask + q * 4096 + h * 128 + pch * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
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

    const long long ngroups = (T + kTok - 1) / kTok;
    const long long g0 = blockIdx.x, gstep = gridDim.x;
    const int nmine = g0 < ngroups ? int((ngroups - 1 - g0) / gstep + 1) : 0;

    // group it goes to stage it % kStages: rows 128 g .. 128 g + 127 of the
    // (T * 32) x 128 view, as two 64-column halves 16 KB apart
    auto load_group = [&](int it) {
        const int s = it % kStages;
        if (err) return;  // no arming without the loads that complete it
        const int row0 = int((g0 + (long long)it * gstep) * 128);
        mbar_expect_tx(bar_full + 8 * s, kStageBytes);
        tma_load_2d(smem_u32(sstage + s * kStageBytes), &tm_x, 0, row0, bar_full + 8 * s);
        tma_load_2d(smem_u32(sstage + s * kStageBytes + kHalfBytes), &tm_x, 64, row0, bar_full + 8 * s);
    };
    if (tid == 0)
        for (int it = 0; it < kStages && it < nmine; ++it) load_group(it);
    __syncwarp();
    {
        const int wg = warp / kGroupWarps;           // takes local groups wg, wg + 2, ...
        const int gtid = tid - wg * kGroupThreads;
        const int gw = warp - wg * kGroupWarps;
        const uint32_t named = 1 + wg;
        float *sred = reinterpret_cast<float *>(base + kOffRed) + wg * kTok * 2;
        const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
        // epilogue mapping: TMEM lane quadrant = token t, lane = head h', column half q
        const int t_in = gw & 3, q = gw >> 2;
        const int h = lane;
        const uint32_t named_tok = 3 + 4 * wg + t_in;  // the two warps holding one token
        uint4 mk[2];
        if (SIGNS) {
#pragma unroll
            for (int k = 0; k < 2; ++k) mk[k] = reinterpret_cast<const uint4 *>(smask)[k * 256 + gtid];
        }

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
                const uint32_t taddr = tmem + (uint32_t(t_in * 32) << 16) + uint32_t(slot * 128 + q * 64);
                tmem_ld32(taddr, r0);
                tmem_ld32(taddr + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    v[k] = __uint_as_float(r0[k]);
                    v[k + 32] = __uint_as_float(r1[k]);
                }
            }
            float mx[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains of three-input maxima
#pragma unroll
            for (int k = 0; k < 64; k += 2) mx[(k >> 1) & 3] = max3(mx[(k >> 1) & 3], fabsf(v[k]), fabsf(v[k + 1]));
            const float wm = warp_max_nonneg(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
            if (lane == 0) sred[t_in * 2 + q] = wm;
            named_sync(named_tok, 64);  // only the two warps that hold this token
            const float amax = fmaxf(sred[t_in * 2], sred[t_in * 2 + 1]);
            const long long t = (g0 + (long long)it * gstep) * kTok + t_in;
            if (t < T) {
                const RowQuant rq = row_quant(amax, qmax);
                uint32_t w[8];
                if (rq.pre == 1.0f)  // the same for the whole warp (one token)
                    quant64<BITS, false>(v, rq, w);
                else
                    quant64<BITS, true>(v, rq, w);
                uint8_t *dst = codes + t * row_bytes + (kDH * h + 64 * q) * BITS / 8;
                if (BITS == 4) {
                    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
                } else {  // 8 groups of 24 bits -> 6 words
                    uint32_t o[6];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        o[3 * g + 0] = w[4 * g] | (w[4 * g + 1] << 24);
                        o[3 * g + 1] = (w[4 * g + 1] >> 8) | (w[4 * g + 2] << 16);
                        o[3 * g + 2] = (w[4 * g + 2] >> 16) | (w[4 * g + 3] << 8);
                    }
#pragma unroll
                    for (int g = 0; g < 3; ++g) reinterpret_cast<uint2 *>(dst)[g] = make_uint2(o[2 * g], o[2 * g + 1]);
                }
                if (h == 0 && q == 0)
                    scales[t] = amax > 0.f ? amax / (float(qmax) * sqrtf(float(kNH))) : 0.f;
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
            if (SIGNS) {
                // the random signs (XOR of bf16 sign bits): chunk gtid + 256 k of the stage
                // is column half k >> 2, head gtid / 8, physical chunk gtid % 8
                uint8_t *st = sstage + s * kStageBytes;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint4 *pc = reinterpret_cast<uint4 *>(st) + gtid + k * kGroupThreads;
                    uint4 xv = *pc;
                    const uint4 mv = mk[k >> 2];
                    xv.x ^= mv.x;
                    xv.y ^= mv.y;
                    xv.z ^= mv.z;
                    xv.w ^= mv.w;
                    *pc = xv;
                }
                fence_proxy_async_cta();
            }
            tc_fence_before();
            named_sync(named, kGroupThreads);
            if (gtid == 0) {
                tc_fence_after();
                // A: K-major, K-steps of 16 are 32 bytes apart within a slab, slabs 16 KB apart.
                // B: MN-major, K rows 128 B apart (16 per K-step: 2 KB), the two 64-column
                //    halves 16 KB apart.
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

template <int BITS, bool SIGNS>
cudaError_t launch_bits(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                        cudaStream_t st) {
    static bool configured[64];
    static EncodeTiledFn enc = nullptr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kern = k_head_mix_tc<BITS, SIGNS>;
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
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
    // x as a (T * 32) x 128 bf16 matrix: row (t, h) = x_t[128 h .. 128 h + 127]
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(kDH), cuuint64_t(T) * kNH};
    const cuuint64_t strides[1] = {cuuint64_t(kDH) * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const long long ngroups = (T + kTok - 1) / kTok;
    long long grid = num_sms();
    if (grid > ngroups) grid = ngroups;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, map, signs, codes, scales, T, status);
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

bool head_mix_tc_supports(int d, int n_heads, int dtype, long long T) {
    // the (T * 32)-row view must fit the tensor map's 32-bit row coordinate
    return dtype == 1 && n_heads == kNH && d == kD && T >= 1 && T <= 0x3FFFFFFLL;
}

cudaError_t launch_head_mix_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                               int bits, cudaStream_t s) {
    if (signs)
        return bits == 4 ? launch_bits<4, true>(x, signs, codes, scales, T, s)
                         : launch_bits<3, true>(x, signs, codes, scales, T, s);
    return bits == 4 ? launch_bits<4, false>(x, signs, codes, scales, T, s)
                     : launch_bits<3, false>(x, signs, codes, scales, T, s);
}

}  // namespace rsq
