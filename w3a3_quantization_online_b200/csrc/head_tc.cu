// head_tc.cu -- per-head randomised Hadamard of attention (QuaRot) on the
// tensor cores: bf16 input, head width d_h in {64, 128}.
//
// Infra Quant II, QuaRot / Method: queries and keys are rotated per head after
// the position transform, v = (I_{n_h} (x) H_{d_h}) diag(s) x / sqrt(d_h), and
// the keys go to a cache quantised per head (one symmetric absmax scale per
// token and head).  QuaRot / Background: H_{d_h} is the Sylvester matrix.
//
// A tile is 128 tokens of one head: the 128 x d_h block X of the activations.
// Its transform is one tcgen05 product
//     V~ = X B,    B = diag(s_h) H_{d_h}     (M = 128, N = K = d_h)
// with s_h the head's signs: B's entries are +-1, exact in bf16, and the
// products are exact; accumulation is fp32 in TMEM.  (Row t of V~ is
// H (s_h o x_t), H being symmetric.)  B is built in shared memory from the
// signs, once per head: each CTA takes a contiguous range of tiles in
// head-major order, so its range spans one or two heads.
//
// Warp roles: warp 0 streams tiles by TMA into a ring of stages, warp 1 issues
// the products into two TMEM slots, warps 2-5 (one per TMEM lane quadrant, one
// token row per thread) run the epilogue: rotation -- V~ / sqrt(d_h) to bf16,
// staged in shared memory and stored by TMA; quantisation -- the (token, head)
// absmax, codes of V~ (codes do not depend on a positive factor), scale
// absmax / sqrt(d_h) / qmax.  The epilogue warps also build the next head's B
// once the product of the current head's last tile has completed.
// Every mbarrier wait is bounded (device status word).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kTok = 128;       // tokens per tile (MMA M)
constexpr int kStages = 3;      // x tiles in flight
constexpr int kEpiWarps = 4;
constexpr int kThreads = (2 + kEpiWarps) * 32;

struct HeadArgs {
    const int8_t *signs;  // d entries, or null (no signs)
    uint8_t *codes;       // quantisation: T rows of d * bits / 8 bytes
    float *scales;        // quantisation: T x n_heads
    int *status;
    long long T;
    int d;
    int n_heads;
    int bits;
    int tiles;            // n_heads * ceil(T / 128)
    int per_cta;          // contiguous tiles per CTA
    int codes_v8;         // codes 32-byte aligned: 256-bit stores
};

template <int DH>
struct HeadLayout {
    static constexpr int kSlabs = DH / 64;                // 64-column slabs of a tile
    static constexpr int kTileBytes = kTok * DH * 2;      // 32 KB (DH = 128) or 16 KB
    static constexpr int kBBytes = DH * DH * 2;           // 32 KB or 8 KB
    static constexpr int kOffX = 0;                       // [kStages] x tiles
    static constexpr int kOffB = kOffX + kStages * kTileBytes;
    static constexpr int kOffOut = kOffB + kBBytes;       // [2] output staging (rotation only)
    static constexpr int kOffBar = kOffOut + 2 * kTileBytes;
    static constexpr int kBytes = kOffBar + 16 * 8 + 16;
    static constexpr int kSmem = kBytes + 1024;
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

enum : int {
    kBarFull = 0,                   // [kStages] tile landed (TMA)
    kBarEmpty = kBarFull + kStages, // [kStages] the product has read the tile (commit)
    kBarTFull = kBarEmpty + kStages,  // [2] product in the TMEM slot (commit)
    kBarTEmpty = kBarTFull + 2,     // [2] TMEM slot read by the epilogue (4 warps)
    kBarB = kBarTEmpty + 2,         // B of the next head built (epilogue)
    kNumBars
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return uint32_t(((chunk ^ (row & 7)) << 4)); }

// B = diag(s_h) H for head h in the K-major SWIZZLE_128B layout the product
// reads: slab k / 64, row n (the output column), 16-byte chunk (k % 64) / 8.
// Stored element (n, k) = s_h[k] * (-1)^popcount(n & k).
template <int DH>
__device__ void build_b(uint8_t *sb, const int8_t *signs, int h, int t0, int nthreads) {
    constexpr int kChunks = DH / 8;  // 16-byte chunks per row of B
    for (int idx = t0; idx < DH * kChunks; idx += nthreads) {
        const int n = idx / kChunks, ck = idx % kChunks;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint16_t hv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int k = 8 * ck + 2 * e + u;
                bool neg = (__popc(n & k) & 1) != 0;
                if (signs && signs[h * DH + k] < 0) neg = !neg;
                hv[u] = neg ? 0xBF80u : 0x3F80u;  // bf16 -1 / +1
            }
            w[e] = uint32_t(hv[0]) | (uint32_t(hv[1]) << 16);
        }
        const int slab = ck / 8, c = ck % 8;
        *reinterpret_cast<uint4 *>(sb + slab * (DH * 128) + n * 128 + swz(n, c)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <int DH, int MODE, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
k_head_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_o, const HeadArgs p) {
    using L = HeadLayout<DH>;
    constexpr int kSlabs = L::kSlabs;
    constexpr uint32_t kTx = uint32_t(L::kTileBytes);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_align1024(smem_raw);
    uint8_t *sb = base + L::kOffB;
    auto xs = [&](int st) { return base + L::kOffX + st * L::kTileBytes; };
    auto os = [&](int b) { return base + L::kOffOut + b * L::kTileBytes; };
    const uint32_t bars = smem_u32(base + L::kOffBar);
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L::kOffBar + 16 * 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tb_per_head = int((p.T + kTok - 1) / kTok);
    const int k0 = int(blockIdx.x) * p.per_cta;
    const int k1 = min(k0 + p.per_cta, p.tiles);
    const int nk = max(k1 - k0, 0);
    auto head_of = [&](int k) { return (k0 + k) / tb_per_head; };
    auto tok0_of = [&](int k) { return ((k0 + k) % tb_per_head) * kTok; };
    int err = 0;
    auto wait = [&](int b, uint32_t ph) {
        if (!mbar_wait(bar(b), ph, err != 0)) err |= kErrMbarTimeout;
    };

    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(bar(i), (i == kBarTEmpty || i == kBarTEmpty + 1) ? kEpiWarps : 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 2 * DH);
        tmem_relinquish();
    }
    if (tid == 32) {
        prefetch_tmap(&tm_x);
        if (MODE == 0) prefetch_tmap(&tm_o);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (nk > 0) build_b<DH>(sb, p.signs, head_of(0), tid, kThreads);  // the first head's B
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ======================= TMA loads
        if (lane == 0) {
#pragma unroll 1
            for (int k = 0; k < nk; ++k) {
                const int st = k % kStages;
                if (k >= kStages) wait(kBarEmpty + st, uint32_t(k / kStages - 1) & 1u);
                if (err) break;  // no arming without the loads that complete it
                mbar_expect_tx(bar(kBarFull + st), kTx);
                const int c0 = head_of(k) * DH, r0 = tok0_of(k);
#pragma unroll
                for (int s = 0; s < kSlabs; ++s)
                    tma_load_2d(smem_u32(xs(st) + s * kTok * 128), &tm_x, c0 + 64 * s, r0, bar(kBarFull + st));
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================= products
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kTok, DH, false, false);
            int nb = 0;  // head changes consumed
#pragma unroll 1
            for (int k = 0; k < nk; ++k) {
                const int st = k % kStages, slot = k & 1;
                if (k > 0 && head_of(k) != head_of(k - 1)) wait(kBarB, uint32_t(nb++) & 1u);  // this head's B
                wait(kBarFull + st, uint32_t(k / kStages) & 1u);
                if (k >= 2) wait(kBarTEmpty + slot, uint32_t((k - 2) >> 1) & 1u);
                tc_fence_after();
                const uint64_t ad = smem_desc_sw128(smem_u32(xs(st)), 1024);
                const uint64_t bd = smem_desc_sw128(smem_u32(sb), 1024);
#pragma unroll
                for (int i = 0; i < DH / 16; ++i) {  // K steps of 16 columns
                    const uint32_t off = uint32_t((i >> 2) * kTok * 128 + (i & 3) * 32) >> 4;
                    const uint32_t boff = uint32_t((i >> 2) * DH * 128 + (i & 3) * 32) >> 4;
                    if (!err) umma_f16(tmem + uint32_t(slot * DH), ad + off, bd + boff, idesc, i != 0);
                }
                if (!err) {
                    umma_commit(bar(kBarEmpty + st));
                    umma_commit(bar(kBarTFull + slot));
                }
            }
        }
        __syncwarp();
    } else {
        // ======================= epilogue: one token row per thread
        const int quad = warp & 3;        // TMEM lane quadrant of this warp
        const int m = 32 * quad + lane;   // token within the tile
        const int et = tid - 64;          // 0 .. 127 among the epilogue threads
        const bool issuer = et == 0;
        const float inv_sqrt = rsqrtf(float(DH));
        const int qmax = MODE == 1 ? (1 << (BITS - 1)) - 1 : 1;
        const long long row_bytes = (long long)p.d * (MODE == 1 ? BITS : 4) / 8;
#pragma unroll 1
        for (int k = 0; k < nk; ++k) {
            const int slot = k & 1, h = head_of(k), r0 = tok0_of(k);
            const long long t = r0 + m;
            wait(kBarTFull + slot, uint32_t(k >> 1) & 1u);
            tc_fence_after();
            if (k + 1 < nk && head_of(k + 1) != h) {
                // the product of this head's last tile has completed: B takes the next head
                build_b<DH>(sb, p.signs, head_of(k + 1), et, kEpiWarps * 32);
                fence_proxy_async_cta();
                named_sync(1, kEpiWarps * 32);
                if (issuer) mbar_arrive(bar(kBarB));
            }
            const uint32_t taddr = tmem + (uint32_t(32 * quad) << 16) + uint32_t(slot * DH);
            if constexpr (MODE == 0) {
                // staging buffer k & 1 is free once the store of tile k - 2 has read it
                if (issuer) bulk_wait_read<1>();
                named_sync(1, kEpiWarps * 32);
                uint8_t *ob = os(slot);
#pragma unroll
                for (int c32 = 0; c32 < DH / 32; ++c32) {
                    uint32_t v[32];
                    tmem_ld32(taddr + 32 * c32, v);
                    tmem_wait_ld();
                    if (c32 == DH / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(kBarTEmpty + slot));
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {  // 16-byte chunks of bf16 output
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            o[e] = pack_bf16x2(__uint_as_float(v[8 * c + 2 * e]) * inv_sqrt,
                                               __uint_as_float(v[8 * c + 2 * e + 1]) * inv_sqrt);
                        const int col = 32 * c32 + 8 * c;  // column within the head
                        *reinterpret_cast<uint4 *>(ob + (col >> 6) * kTok * 128 + m * 128 + swz(m, (col & 63) >> 3)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                fence_proxy_async_cta();
                named_sync(1, kEpiWarps * 32);
                if (issuer) {
#pragma unroll
                    for (int s = 0; s < kSlabs; ++s)
                        if (!err) tma_store_2d(&tm_o, smem_u32(ob + s * kTok * 128), h * DH + 64 * s, r0);
                    bulk_commit();
                }
            } else {
                // two reads of the slot: the absmax, then the codes (32 columns at a time)
                float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c32 = 0; c32 < DH / 32; ++c32) {
                    uint32_t v[32];
                    tmem_ld32(taddr + 32 * c32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            am[e] = max3(am[e], fabsf(__uint_as_float(v[i + 2 * e])),
                                         fabsf(__uint_as_float(v[i + 2 * e + 1])));
                }
                const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
                const RowQuant rq = row_quant(amax, qmax);
                uint8_t *dst = p.codes + t * row_bytes + (long long)h * DH * BITS / 8;
#pragma unroll
                for (int g = 0; g < DH / 64; ++g) {  // 64 codes at a time
                    uint32_t words[2 * BITS];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t v[32];
                        tmem_ld32(taddr + 64 * g + 32 * half, v);
                        tmem_wait_ld();
                        if (g == DH / 64 - 1 && half == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar(kBarTEmpty + slot));  // the slot may take tile k + 2
                        }
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * q4 + e]);
                            const uint32_t w = pack8_fast<BITS>(f, rq.inv, rq.pre, true);
                            const int q = 4 * half + q4;  // group of 8 codes within the 64
                            if (BITS == 4) {
                                words[q] = w;
                            } else {  // 8 codes = one little-endian 24-bit group
                                const int bit = 24 * q;
                                if (bit % 32 == 0) {
                                    words[bit / 32] = w;
                                } else {
                                    words[bit / 32] |= w << (bit % 32);
                                    if (bit % 32 > 8) words[bit / 32 + 1] = w >> (32 - bit % 32);
                                }
                            }
                        }
                    }
                    if (t < p.T) {
                        uint8_t *gd = dst + g * 8 * BITS;
                        if (BITS == 4) {
                            if (p.codes_v8) {
                                st_global_v8(gd, words);
                            } else {
                                reinterpret_cast<uint4 *>(gd)[0] = make_uint4(words[0], words[1], words[2], words[3]);
                                reinterpret_cast<uint4 *>(gd)[1] = make_uint4(words[4], words[5], words[6], words[7]);
                            }
                        } else {
                            reinterpret_cast<uint2 *>(gd)[0] = make_uint2(words[0], words[1]);
                            reinterpret_cast<uint2 *>(gd)[1] = make_uint2(words[2], words[3]);
                            reinterpret_cast<uint2 *>(gd)[2] = make_uint2(words[4], words[5]);
                        }
                    }
                }
                if (t < p.T) {
                    p.scales[t * p.n_heads + h] = amax > 0.f ? amax * inv_sqrt / float(qmax) : 0.f;
                }
            }
        }
        if (MODE == 0 && issuer) bulk_wait0();
    }

    tc_fence_before();
    if (__syncthreads_or(err)) drain_delay();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 2 * DH);
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(p.status, err);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

bool make_map(CUtensorMap *mp, const void *ptr, long long T, int d) {
    static EncodeTiledFn enc = nullptr;
    if (!enc) {
        void *q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) != cudaSuccess ||
            res != cudaDriverEntryPointSuccess)
            return false;
        enc = reinterpret_cast<EncodeTiledFn>(q);
    }
    const cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(d) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(kTok)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DH, int MODE, int BITS>
cudaError_t launch_typed(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales, long long T,
                         int d, int n_heads, int *status, cudaStream_t s) {
    using L = HeadLayout<DH>;
    auto kern = k_head_tc<DH, MODE, BITS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    CUtensorMap mx, mo;
    if (!make_map(&mx, x, T, d)) return cudaErrorInvalidValue;
    if (MODE == 0 && !make_map(&mo, x_out, T, d)) return cudaErrorInvalidValue;
    if (MODE == 1) mo = mx;  // unused
    HeadArgs a;
    a.signs = signs;
    a.codes = codes;
    a.scales = scales;
    a.status = status;
    a.T = T;
    a.d = d;
    a.n_heads = n_heads;
    a.bits = BITS;
    const long long tb = (T + kTok - 1) / kTok;
    a.tiles = int(tb * n_heads);
    long long grid = num_sms();
    if (grid > a.tiles) grid = a.tiles;
    a.per_cta = int((a.tiles + grid - 1) / grid);
    grid = (a.tiles + a.per_cta - 1) / a.per_cta;
    a.codes_v8 = (reinterpret_cast<uintptr_t>(codes) & 31u) == 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mx, mo, a);
    if (e == cudaSuccess) count_launch();
    return e;
}

template <int DH>
cudaError_t launch_dh(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales, long long T,
                      int d, int n_heads, int bits, bool quant, int *status, cudaStream_t s) {
    if (!quant) return launch_typed<DH, 0, 4>(x, signs, x_out, nullptr, nullptr, T, d, n_heads, status, s);
    return bits == 4 ? launch_typed<DH, 1, 4>(x, signs, nullptr, codes, scales, T, d, n_heads, status, s)
                     : launch_typed<DH, 1, 3>(x, signs, nullptr, codes, scales, T, d, n_heads, status, s);
}

}  // namespace

bool head_tc_supports(int d, int n_heads, int dtype, long long T) {
    if (dtype != 1 || n_heads < 1 || d % n_heads || T < 1 || T > 0x7FFFFFFFLL) return false;
    const int dh = d / n_heads;
    return (dh == 64 || dh == 128) && (long long)n_heads * ((T + kTok - 1) / kTok) <= 0x7FFFFFFFLL;
}

cudaError_t launch_head_tc(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales,
                           long long T, int d, int n_heads, int bits, bool quant, cudaStream_t s) {
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    return d / n_heads == 128 ? launch_dh<128>(x, signs, x_out, codes, scales, T, d, n_heads, bits, quant, status, s)
                              : launch_dh<64>(x, signs, x_out, codes, scales, T, d, n_heads, bits, quant, status, s);
}

}  // namespace rsq
