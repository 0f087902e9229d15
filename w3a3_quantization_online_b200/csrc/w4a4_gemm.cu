// w4a4_gemm.cu -- the INT4 consumer GEMM of the quantised activations (W4A4).
//
// Infra Quant II, QuaRot / Method: the INT4 GEMM's INT32 output is converted to
// 16-bit float and multiplied by the activation's per-row scale and the weight's
// per-column scale.  Here Y[t][n] = round16(float(acc[t][n]) * sa[t] * sw[n])
// with acc = qa qw^T exact in int32 (|acc| <= 64 K), qa the packed per-token
// activation codes written by the quantising entry points and qw the packed
// per-output-channel weight codes (element 2i in the low nibble of byte i,
// two's complement, any 4-bit value).
//
// Design (B200, sm_100a): one CTA per 128 x 256 output tile, 10 warps.
//  * Warp 0 (one thread): TMA loads of the packed tiles, 128 rows of A and 256
//    rows of B by 64 bytes (128 K values), into a 3-stage ring.
//  * Warps 2-9: unpack.  A 16-byte chunk of packed codes (32 values) becomes
//    two 16-byte chunks of int8 in the SWIZZLE_128B K-major layout of a
//    tcgen05 operand (nibbles masked into bytes, sign-extended by a multiply
//    that cannot carry across bytes, even/odd elements interleaved by byte
//    permutes); four consecutive threads take the four chunks of one packed
//    row, so both the reads and the swizzled writes are free of bank
//    conflicts.  2-stage ring of unpacked operands.
//  * Warp 1 (one thread): tcgen05.mma kind::i8 (s8 x s8 -> s32, M = 128,
//    N = 256, K = 32), four per stage, accumulating in 256 TMEM columns.
//  * Epilogue, warps 2-9: TMEM -> registers, float(acc) * sa * sw, rounded to
//    fp16 or bf16 into a swizzled staging tile, written by TMA (4 slabs of 64
//    columns); optionally the raw int32 accumulators as well.
//  * Prepared weights (w4a4_gemm_s8w): the weight codes, unpacked once to
//    int8 by w4a4_prepare_weights, are TMA-loaded straight into the SWIZZLE_128B
//    K-major operand layout; only the activation codes are unpacked, and the
//    ring of operand stages is four deep (the packed ring holds A alone).
//    Without it every 128-row M tile unpacks the whole weight again: two thirds
//    of the unpack work and of its shared-memory traffic.
// Every mbarrier wait is bounded; a timeout sets a bit in the device status
// word, no further asynchronous work is issued, and the CTA drains what is in
// flight before freeing TMEM.
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kPA = kBM * kBK / 2;  // packed A bytes per stage (8 KB)
constexpr int kPB = kBN * kBK / 2;  // packed B bytes per stage (16 KB)
constexpr int kUA = kBM * kBK;      // unpacked A bytes per stage (16 KB)
constexpr int kUB = kBN * kBK;      // unpacked B bytes per stage (32 KB)
constexpr int kUnpackWarps = 8;
constexpr int kEpiWarps = 4;                   // one per TMEM lane quadrant
constexpr int kFirstEpiWarp = 2 + kUnpackWarps;
constexpr int kGThreads = (2 + kUnpackWarps + kEpiWarps) * 32;
constexpr int kGTmemCols = 512;                // two 256-column int32 accumulators
constexpr int kSlabOut = kBM * 128;            // one 64-column output slab of 16-bit values (16 KB)

// PREP = false: packed A and B ring of 3, operand ring of 2.  PREP = true: the
// int8 weights go by TMA into the operand ring, whose stages hold both
// operands: packed A ring of 4, operand ring of 3.  Two 16 KB output staging
// slabs for the epilogue.
template <bool PREP>
struct GemmCfg {
    static constexpr int kP = PREP ? 4 : 3, kU = PREP ? 3 : 2;  // ring depths
    static constexpr int kPStage = PREP ? kPA : kPA + kPB;
    static constexpr int kOffPk = 0;                                    // packed ring
    static constexpr int kOffUn = (kOffPk + kP * kPStage + 1023) / 1024 * 1024;  // operand ring
    static constexpr int kOffOut = kOffUn + kU * (kUA + kUB);           // 2 output staging slabs
    static constexpr int kOffBar = kOffOut + 2 * kSlabOut;
    static constexpr int kPFull = 0, kPEmpty = kPFull + kP, kUFull = kPEmpty + kP, kUEmpty = kUFull + kU;
    static constexpr int kAccFull = kUEmpty + kU, kAccEmpty = kAccFull + 2, kGBars = kAccEmpty + 2;
    static constexpr int kOffTm = kOffBar + kGBars * 8;
    static constexpr int kGSmem = kOffTm + 16 + 1024;
    static_assert(kOffUn % 1024 == 0 && (kUA + kUB) % 1024 == 0 && kOffOut % 1024 == 0, "swizzle atoms");
    static_assert(kGSmem <= 232448, "shared memory per CTA");
};

struct GemmArgs {
    const float *sa;
    const float *sw;
    int32_t *acc;  // optional raw accumulators (T x N)
    int *status;
    long long T;
    int N;
    int K;
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return uint32_t(((chunk ^ (row & 7)) << 4)); }

// Instruction descriptor, kind::i8: s8 x s8 -> s32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
    return (2u << 4)      // D format: s32
           | (1u << 7)    // A format: signed 8-bit
           | (1u << 10)   // B format: signed 8-bit
           | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 8 packed 4-bit codes (one word) -> 8 int8 (two words), element order kept.
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t &o0, uint32_t &o1) {
    uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    lo |= (lo & 0x08080808u) * 0x1Eu;  // bit 3 of a byte -> bits 4-7 of the same byte
    hi |= (hi & 0x08080808u) * 0x1Eu;
    o0 = prmt(lo, hi, 0x5140u);        // elements 0, 1, 2, 3
    o1 = prmt(lo, hi, 0x7362u);        // elements 4, 5, 6, 7
}

// One packed row chunk (16 bytes: K values 32 c .. 32 c + 31 of row r) -> the
// two unpacked 16-byte chunks 2 c and 2 c + 1 of row r.
__device__ __forceinline__ void unpack_chunk(const uint8_t *pk, uint8_t *un, int r, int c) {
    const uint4 p = *reinterpret_cast<const uint4 *>(pk + r * 64 + c * 16);
    uint32_t o[8];
    unpack8(p.x, o[0], o[1]);
    unpack8(p.y, o[2], o[3]);
    unpack8(p.z, o[4], o[5]);
    unpack8(p.w, o[6], o[7]);
    uint8_t *row = un + r * 128;
    *reinterpret_cast<uint4 *>(row + swz(r, 2 * c)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4 *>(row + swz(r, 2 * c + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
}

template <class OUT>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
    return pack_bf16x2(a, b);
}

template <class OUT, bool PREP>
__global__ void __launch_bounds__(kGThreads, 1)
k_w4a4_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
            const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
    using C = GemmCfg<PREP>;
    constexpr int kP = C::kP, kU = C::kU, kPStage = C::kPStage, kOffPk = C::kOffPk, kOffUn = C::kOffUn;
    constexpr int kOffOut = C::kOffOut, kOffBar = C::kOffBar, kOffTm = C::kOffTm;
    constexpr int kPFull = C::kPFull, kPEmpty = C::kPEmpty, kUFull = C::kUFull, kUEmpty = C::kUEmpty;
    constexpr int kAccFull = C::kAccFull, kAccEmpty = C::kAccEmpty, kGBars = C::kGBars;
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *base = smem_align1024(gsm_raw);
    const uint32_t bars = smem_u32(base + kOffBar);
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffTm);
    auto pk_a = [&](int s) { return base + kOffPk + s * kPStage; };
    auto pk_b = [&](int s) { return base + kOffPk + s * kPStage + kPA; };  // packed weights only
    auto un_a = [&](int s) { return base + kOffUn + s * (kUA + kUB); };
    auto un_b = [&](int s) { return base + kOffUn + s * (kUA + kUB) + kUA; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KS = p.K / kBK;
    const int ntn = (p.N + kBN - 1) / kBN;
    const long long ntiles = (long long)((p.T + kBM - 1) / kBM) * ntn;
    // this CTA's output tiles: blockIdx.x, + gridDim.x, ... (n fastest: consecutive
    // CTAs share the activation block in L2)
    const int nmine = blockIdx.x < ntiles ? int((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
    auto tile_mn = [&](int i, long long &m0, int &n0) {
        const long long tile = blockIdx.x + (long long)i * gridDim.x;
        m0 = (tile / ntn) * kBM;
        n0 = int(tile % ntn) * kBN;
    };
    int err = 0;
    auto wait = [&](int b, uint32_t ph) {
        if (!mbar_wait(bar(b), ph, err != 0)) err |= kErrMbarTimeout;
    };

    if (tid == 0) {
        for (int i = 0; i < kGBars; ++i)
            mbar_init(bar(i), (i >= kPEmpty && i < kPEmpty + kP) ? kUnpackWarps
                              : (i >= kUFull && i < kUFull + kU) ? kUnpackWarps + (PREP ? 1 : 0)  // + the weight load
                              : (i >= kAccEmpty && i < kAccEmpty + 2) ? kEpiWarps
                              : 1);
        fence_mbar_init();
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_y);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kGTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The rings run on one K-step counter g across all of this CTA's tiles.
    if (warp == 0) {
        // ---- TMA producer
        if (lane == 0) {
            int g = 0;
            for (int i = 0; i < nmine && !err; ++i) {
                long long m0;
                int n0;
                tile_mn(i, m0, n0);
                for (int ks = 0; ks < KS; ++ks, ++g) {
                    const int s = g % kP;
                    wait(kPEmpty + s, uint32_t((g / kP) & 1) ^ 1u);
                    if (err) break;  // no arming without the loads that complete it
                    mbar_expect_tx(bar(kPFull + s), uint32_t(kPStage));
                    tma_load_2d(smem_u32(pk_a(s)), &tm_a, ks * (kBK / 2), int(m0), bar(kPFull + s));
                    if (PREP) {
                        // int8 weights straight into the operand stage, once the product has freed it
                        const int u = g % kU;
                        wait(kUEmpty + u, uint32_t((g / kU) & 1) ^ 1u);
                        if (err) break;
                        mbar_expect_tx(bar(kUFull + u), uint32_t(kUB));
                        tma_load_2d(smem_u32(un_b(u)), &tm_b, ks * kBK, n0, bar(kUFull + u));
                    } else {
                        tma_load_2d(smem_u32(pk_b(s)), &tm_b, ks * (kBK / 2), n0, bar(kPFull + s));
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- tensor-core issue: tile i accumulates in TMEM columns [256 (i & 1), +256)
        if (lane == 0) {
            const uint32_t idesc = idesc_s8_s32(kBM, kBN);
            int g = 0;
            for (int i = 0; i < nmine; ++i) {
                const int ab = i & 1;
                wait(kAccEmpty + ab, uint32_t((i >> 1) & 1) ^ 1u);  // its previous tile has been read out
                tc_fence_after();
                for (int ks = 0; ks < KS; ++ks, ++g) {
                    const int u = g % kU;
                    wait(kUFull + u, uint32_t((g / kU) & 1));
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(smem_u32(un_a(u)), 1024);
                    const uint64_t bd = smem_desc_sw128(smem_u32(un_b(u)), 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k)  // K steps of 32 int8 = 32 bytes
                        if (!err) umma_i8(tmem + uint32_t(256 * ab), ad + uint64_t((k * 32) >> 4),
                                          bd + uint64_t((k * 32) >> 4), idesc, (ks | k) != 0);
                    if (!err) umma_commit(bar(kUEmpty + u));
                }
                if (!err) umma_commit(bar(kAccFull + ab));
            }
        }
        __syncwarp();
    } else if (warp < kFirstEpiWarp) {
        // ---- unpack
        const int u_tid = tid - 64;  // 0..255
        int g = 0;
        for (int i = 0; i < nmine; ++i) {
            for (int ks = 0; ks < KS; ++ks, ++g) {
                const int s = g % kP, u = g % kU;
                wait(kPFull + s, uint32_t((g / kP) & 1));
                wait(kUEmpty + u, uint32_t((g / kU) & 1) ^ 1u);
                const uint8_t *pa = pk_a(s), *pb = PREP ? nullptr : pk_b(s);
                uint8_t *ua = un_a(u), *ub = un_b(u);
#pragma unroll
                for (int j = 0; j < 2; ++j) {  // A: 512 chunks
                    const int c = u_tid + 256 * j;
                    unpack_chunk(pa, ua, c >> 2, c & 3);
                }
                if (!PREP) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {  // B: 1024 chunks
                        const int c = u_tid + 256 * j;
                        unpack_chunk(pb, ub, c >> 2, c & 3);
                    }
                }
                fence_proxy_async_cta();  // unpacked operands (generic writes) -> tensor core (async proxy)
                __syncwarp();
                if (lane == 0 && !err) {
                    mbar_arrive(bar(kPEmpty + s));
                    mbar_arrive(bar(kUFull + u));
                }
            }
        }
    } else {
        // ---- epilogue: TMEM lane quadrant q (one output row per thread), 64-column
        // slabs through two staging buffers, each written back by one TMA store
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const bool leader = warp == kFirstEpiWarp && lane == 0;
        int slabs_done = 0;
        for (int i = 0; i < nmine; ++i) {
            const int ab = i & 1;
            long long m0;
            int n0;
            tile_mn(i, m0, n0);
            const long long row = m0 + r;
            const float sa = row < p.T ? p.sa[row] : 0.f;
            wait(kAccFull + ab, uint32_t((i >> 1) & 1));
            __syncwarp();
            tc_fence_after();
#pragma unroll 1
            for (int sl = 0; sl < kBN / 64; ++sl, ++slabs_done) {
                const int sb = slabs_done & 1;
                uint8_t *slab = base + kOffOut + sb * kSlabOut;
                // staging buffer sb is free once the store issued from it two slabs ago has read it
                if (leader) bulk_wait_read<1>();
                named_sync(1, kEpiWarps * 32);
                if (n0 + 64 * sl < p.N) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {  // 32-column blocks
                        uint32_t v[32];
                        tmem_ld32(tmem + (uint32_t(32 * q) << 16) + uint32_t(256 * ab + 64 * sl + 32 * h), v);
                        tmem_wait_ld();
                        const int c0 = 64 * sl + 32 * h;  // first column of the block within the tile
                        if (p.acc && row < p.T) {
                            int32_t *dst = p.acc + row * p.N + n0 + c0;
                            if (n0 + c0 + 32 <= p.N) {
#pragma unroll
                                for (int e = 0; e < 32; e += 4)
                                    *reinterpret_cast<int4 *>(dst + e) =
                                        make_int4(int(v[e]), int(v[e + 1]), int(v[e + 2]), int(v[e + 3]));
                            } else {
                                for (int e = 0; e < 32; ++e)
                                    if (n0 + c0 + e < p.N) dst[e] = int(v[e]);
                            }
                        }
                        uint32_t o[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int c = n0 + c0 + 2 * e;
                            const float w0 = c < p.N ? __ldg(p.sw + c) : 0.f;
                            const float w1 = c + 1 < p.N ? __ldg(p.sw + c + 1) : 0.f;
                            o[e] = pack2<OUT>(float(int(v[2 * e])) * sa * w0, float(int(v[2 * e + 1])) * sa * w1);
                        }
                        uint8_t *srow = slab + r * 128;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4 *>(srow + swz(r, 4 * h + c)) =
                                make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                    }
                }
                fence_proxy_async_cta();  // staged outputs (generic writes) -> TMA store (async proxy)
                named_sync(1, kEpiWarps * 32);
                if (leader) {
                    if (!err && n0 + 64 * sl < p.N) tma_store_2d(&tm_y, smem_u32(slab), n0 + 64 * sl, int(m0));
                    bulk_commit();
                }
            }
            // every TMEM load of this tile is complete: the accumulator may take tile i + 2
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !err) mbar_arrive(bar(kAccEmpty + ab));
        }
        if (leader) bulk_wait0();
    }

    tc_fence_before();
    if (__syncthreads_or(err)) drain_delay();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kGTmemCols);
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(p.status, err);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(q);
    }
    return fn;
}

bool make_map_2d(CUtensorMap *mp, const void *ptr, CUtensorMapDataType dt, int esize, long long rows, long long cols,
                 int box_cols, int box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(cols) * esize};
    const cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(mp, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool w4a4_gemm_supports(long long T, int N, int K) {
    return T >= 1 && T <= 65535LL * kBM && N >= 8 && N % 8 == 0 && K >= kBK && K % kBK == 0 && K <= 65536;
}

cudaError_t launch_w4a4_gemm(const uint8_t *codes_a, const float *sa, const void *w, bool w_prepared, const float *sw,
                             void *y, int32_t *acc, long long T, int N, int K, int out_f16, cudaStream_t s) {
    static bool configured[4][64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    using KernFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, GemmArgs);
    const KernFn kern = w_prepared ? (out_f16 ? k_w4a4_gemm<__half, true> : k_w4a4_gemm<__nv_bfloat16, true>)
                                   : (out_f16 ? k_w4a4_gemm<__half, false> : k_w4a4_gemm<__nv_bfloat16, false>);
    const int smem = w_prepared ? GemmCfg<true>::kGSmem : GemmCfg<false>::kGSmem;
    const int variant = (w_prepared ? 2 : 0) + (out_f16 ? 1 : 0);
    if (dev >= 0 && dev < 64 && !configured[variant][dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured[variant][dev] = true;
    }
    CUtensorMap ma, mb, my;
    const bool ok_b = w_prepared
        // int8 weights: 128-byte rows of K values, swizzled as the operand
        ? make_map_2d(&mb, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B)
        : make_map_2d(&mb, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, K / 2, kBK / 2, kBN, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!make_map_2d(&ma, codes_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, K / 2, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !ok_b ||
        !make_map_2d(&my, y, out_f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, T, N, 64,
                     kBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    GemmArgs a;
    a.sa = sa;
    a.sw = sw;
    a.acc = acc;
    a.status = status;
    a.T = T;
    a.N = N;
    a.K = K;
    // persistent: one CTA per SM (at most one per output tile)
    const long long ntiles = ((T + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    long long grid = num_sms();
    if (grid > ntiles) grid = ntiles;
    kern<<<unsigned(grid), kGThreads, smem, s>>>(ma, mb, my, a);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

// The weight codes unpacked once to int8 (sign-extended 4-bit values, element
// order kept): 16 packed bytes -> 32 int8 per thread, grid-stride.
__global__ void __launch_bounds__(256)
k_w4a4_unpack_weights(const uint4 *__restrict__ codes, uint4 *__restrict__ w, long long n16) {
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n16; i += (long long)gridDim.x * 256) {
        const uint4 pk = codes[i];
        uint32_t o[8];
        unpack8(pk.x, o[0], o[1]);
        unpack8(pk.y, o[2], o[3]);
        unpack8(pk.z, o[4], o[5]);
        unpack8(pk.w, o[6], o[7]);
        w[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
        w[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

cudaError_t launch_w4a4_unpack_weights(const uint8_t *codes_w, int8_t *w_s8, int N, int K, cudaStream_t s) {
    const long long n16 = (long long)N * (K / 2) / 16;  // K % 128 == 0: whole 16-byte chunks
    long long grid = (n16 + 255) / 256;
    const long long cap = 8LL * num_sms();
    if (grid > cap) grid = cap;
    k_w4a4_unpack_weights<<<unsigned(grid), 256, 0, s>>>(reinterpret_cast<const uint4 *>(codes_w),
                                                         reinterpret_cast<uint4 *>(w_s8), n16);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace rsq
