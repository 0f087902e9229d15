// align_tc.cu -- tensor-core (tcgen05) residual subspace alignment fused with
// the weight-free RMSNorm and the per-token symmetric quantiser, bf16 I/O.
//
// ReSpinQuant paper notes, key design 3: y = Q^T x (D -> r), z = M y,
// x_out = x + Q z.  Infra Quant II, QuaRot / Method: scale-free RMSNorm in FP32
// and per-token symmetric absmax quantisation (SpinQuant / Motivation gives
// alpha = max|X| / (2^(N-1) - 1)).
//
// Design (B200, sm_100a):
//  * A cluster of CS CTAs splits the hidden dimension: CTA c owns columns
//    [512 c, 512 c + 512) and keeps its 512 x 32 slice of Q resident in shared
//    memory for the whole persistent kernel.  Every token tile (up to 128 rows)
//    is read from HBM exactly once by TMA and stays in shared memory until its
//    x_out has been written.
//  * Both rank-32 contractions run on the 5th-generation tensor cores with fp32
//    accumulators in TMEM.  x is exact in bf16; Q and z are split into bf16
//    high and low parts (Q = Q_hi + Q_lo), which keeps the products accurate to
//    about 2^-16 relative:
//        y   = x [Q_hi | Q_lo]              (M=128, N=64, K=512 per CTA)
//        c   = z_hi Q_hi^T + z_hi Q_lo^T + z_lo Q_hi^T   (M=128, N=4x128, K=96)
//    The same shared-memory Q buffer serves as the MN-major B operand of the
//    first product and the K-major B operand of the second.
//  * Sixteen warps, four per TMEM lane quadrant, each on 128 columns of its 32
//    rows.  Thread 0 also issues the first product (following the tile's slabs
//    as they land) and an L2 prefetch of the next tile; a warp of the last
//    column part issues the second product; the last warp issues the x_out
//    stores and the next tile's loads.
//  * Cross-CTA exchange.  After one cluster barrier the CTA that owns 128/CS
//    token rows reads their CS partial projections through distributed shared
//    memory, applies the r x r matrix M and copies z (split hi/lo) into every
//    CTA's operand buffer by bulk copy, counted on a local mbarrier there.  The
//    row statistics (sum of squares, absmax) are pushed with st.async to the
//    row's owner, which forms the row quantiser and pushes it back to all CTAs.
//    Every exchange needs all CTAs of the cluster, so one buffer per exchange
//    suffices: no CTA can run a whole tile ahead of another.
//  * x_out = x + c is formed in fp32, rounded to bf16 in place in the tile
//    buffer and written back by TMA, slab by slab; each slab takes the next
//    tile as soon as its store has read it, so the load overlaps the statistics
//    exchange and the codes.  The fp32 value goes back to TMEM, from which the
//    codes are computed once the row quantiser arrives.
//  * Programmatic dependent launch: the kernel lets the next kernel of the
//    stream start at once, and stages its own Q slice and M while the previous
//    kernel may still run; it waits for that kernel before touching x or any
//    output.
// Every mbarrier wait is bounded; a timeout sets a bit in the device status
// word and the kernel keeps its barrier sequence so that no CTA is left
// waiting; after a failed wait a thread issues no further asynchronous work,
// and the CTA drains what is in flight before freeing TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kTileM = 128;                  // token rows per tile (MMA M)
constexpr int kCols = 512;                   // hidden columns owned by one CTA
constexpr int kSlabCols = 64;                // bf16 columns per 128-byte swizzle row
constexpr int kSlabs = kCols / kSlabCols;    // 8
constexpr int kSlabBytes = kTileM * 128;     // 16 KB
constexpr int kXBytes = kSlabs * kSlabBytes; // 128 KB
constexpr int kQBytes = kCols * 128;         // 64 KB: 512 rows x [Q_hi(32) | Q_lo(32)] bf16
constexpr int kZBytes = kTileM * 128;        // 16 KB: partial y (fp32) / z hi|lo (bf16), per row
constexpr int kParts = 4;                    // consumer warps per TMEM lane quadrant (column parts)
constexpr int kConsumerWarps = 4 * kParts;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers;
constexpr int kTmemCols = 512;
constexpr int kPartCols = kCols / kParts;    // columns per consumer thread (128)
constexpr int kMma2Warp = 4 * (kParts - 1);  // first warp of the last column part

struct AlignTcArgs {
    const float *Q;
    const float *M;
    uint8_t *codes;
    float *scales;
    int *status;
    long long T;
    int D;
    int r;
    int rows_per_tile;
    int tiles_per_cluster;
    int codes_v8;  // codes pointer is 32-byte aligned: 256-bit stores
    float eps;
};

// mbarriers (each completes once per tile)
enum : int {
    kBarLd = 0,               // kSlabs: x slab landed (TMA)
    kBarY = kBarLd + kSlabs,  // partial projection in TMEM (commit)
    kBarZ,                    // z of all rows in the operand buffer (local owner warps + bulk copies)
    kBarC,                    // 4: correction columns [128 q, 128 q + 128) in TMEM (commit)
    kBarSt = kBarC + 4,       // owner: row statistics of all CTAs pushed (st.async)
    kBarPrm,                  // row quantisers of all rows pushed (st.async)
    kNumBars
};

template <int CS>
struct Layout {
    static constexpr int kTokPerOwner = kTileM / CS;
    static constexpr int kOffX = 0;
    static constexpr int kOffQ = kOffX + kXBytes;
    static constexpr int kOffZ = kOffQ + kQBytes;
    static constexpr int kOffM = kOffZ + kZBytes;            // M^T, 32 x 32 fp32, zero padded
    static constexpr int kOffSt = kOffM + 32 * 32 * 4;       // owner: [source CTA][own row] (ss, amax), 16 B
    static constexpr int kOffPrm = kOffSt + CS * kTokPerOwner * 16;  // per row: (inv, pre)
    static constexpr int kOffLoc = kOffPrm + kTileM * 8;     // column-part partial statistics, 16 B
    static constexpr int kOffBar = kOffLoc + (kParts - 1) * kTileM * 16;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffTmem + 16;
    static constexpr int kSmem = kBytes + 1024;  // slack for 1024-byte alignment
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // SWIZZLE_128B chunk position
    return uint32_t(((chunk ^ (row & 7)) << 4));
}

// Opaque copy: keeps the compiler from hoisting descriptor arithmetic out of the
// tile loop (which would pin dozens of 64-bit descriptors in registers).
__device__ __forceinline__ uint64_t opaque(uint64_t v) {
    asm volatile("mov.b64 %0, %0;" : "+l"(v));
    return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t *>(&h);
}

__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

// x_out = x + c for one 32-column block of row m: updates the fp32 values in
// v (TMEM copy), writes bf16 x_out in place over x, accumulates the sum of
// squares (pairs, fp32) and the absmax (four independent partial maxima).
__device__ __forceinline__ void xout_block(uint32_t (&v)[32], uint8_t *rowp, int m, int chunk0, float2 &s2,
                                           float (&am)[4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint8_t *cp = rowp + swz(m, chunk0 + q);
        const uint4 u = *reinterpret_cast<const uint4 *>(cp);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 xv = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
            const float2 cv = make_float2(__uint_as_float(v[q * 8 + 2 * e]), __uint_as_float(v[q * 8 + 2 * e + 1]));
            const float2 y = add2(xv, cv);
            v[q * 8 + 2 * e] = __float_as_uint(y.x);
            v[q * 8 + 2 * e + 1] = __float_as_uint(y.y);
            s2 = fma2(y, y, s2);
            am[e] = max3(am[e], fabsf(y.x), fabsf(y.y));
            o[e] = pack_bf16x2(y.x, y.y);
        }
        *reinterpret_cast<uint4 *>(cp) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Wait until at most n (0..7) of this thread's bulk groups still read shared memory.
__device__ __forceinline__ void bulk_wait_read_n(int n) {
    switch (n) {
        case 0: bulk_wait_read<0>(); break;
        case 1: bulk_wait_read<1>(); break;
        case 2: bulk_wait_read<2>(); break;
        case 3: bulk_wait_read<3>(); break;
        case 4: bulk_wait_read<4>(); break;
        case 5: bulk_wait_read<5>(); break;
        case 6: bulk_wait_read<6>(); break;
        default: bulk_wait_read<7>(); break;
    }
}

// Codes of one 32-column block (INT4: 4 words, INT3: 3 words).
template <int BITS>
__device__ __forceinline__ void code_block(const uint32_t (&v)[32], const RowQuant &rq, uint32_t *words) {
    uint32_t g[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[gi * 8 + e]);
        // the row factor pre (1, or 2^64 for a tiny row) is always applied: one
        // packed multiply per pair is cheaper than a per-element predicate
        g[gi] = pack8_fast<BITS>(f, rq.inv, rq.pre, true);
    }
    if (BITS == 4) {
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) words[gi] = g[gi];
    } else {
        words[0] = g[0] | (g[1] << 24);
        words[1] = (g[1] >> 8) | (g[2] << 16);
        words[2] = (g[2] >> 16) | (g[3] << 8);
    }
}

template <int CS, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
k_align_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xo,
           const AlignTcArgs p) {
    using L = Layout<CS>;
    constexpr int TPO = L::kTokPerOwner;    // token rows owned by each CTA: one consumer warp each
    static_assert(CS * kCols <= 16384 && TPO <= kConsumerWarps && CS * TPO == kTileM, "cluster shape");
    static_assert(TPO * CS <= kConsumers, "owner statistics threads");
    constexpr int kZTx = (CS - 1) * TPO * 128;  // z rows arriving from the other CTAs

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_align1024(smem_raw);
    uint8_t *sx = base + L::kOffX;
    uint8_t *sq = base + L::kOffQ;
    uint8_t *sz = base + L::kOffZ;
    float *sm = reinterpret_cast<float *>(base + L::kOffM);
    uint8_t *sst = base + L::kOffSt;
    uint8_t *sprm = base + L::kOffPrm;
    uint8_t *sloc = base + L::kOffLoc;
    const uint32_t bars = smem_u32(base + L::kOffBar);
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L::kOffTmem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
    const int col0 = int(crank) * kCols;
    const int r = p.r;
    constexpr bool kQuant = BITS > 0;  // BITS = 0: alignment only (x_out), no norm / codes
    const int qmax = kQuant ? (1 << (BITS - 1)) - 1 : 1;
    const long long row_bytes = (long long)p.D * BITS / 8;
    const int R = p.rows_per_tile;
    int err = 0;

    // programmatic dependent launch: the next kernel of the stream may start and
    // stage its constants now; it waits for this grid before it touches data
    asm volatile("griddepcontrol.launch_dependents;");
    auto tile_t0 = [&](int it) { return ((long long)cid + (long long)it * ncl) * R; };
    auto has_tile = [&](int it) { return it < p.tiles_per_cluster && tile_t0(it) < p.T; };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), i == kBarZ ? 1 + TPO : 1);
        fence_mbar_init();
        // the pushed exchanges of the first tile (each barrier is re-armed by its
        // waiter once the previous phase has completed)
        if (has_tile(0)) {
            mbar_expect_tx(bar(kBarZ), uint32_t(kZTx));
            if (kQuant) {
                mbar_expect_tx(bar(kBarSt), uint32_t(CS * TPO * 16));
                mbar_expect_tx(bar(kBarPrm), uint32_t(kTileM * 8));
            }
        }
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_xo);
    }

    // Q slice -> shared memory as [Q_hi | Q_lo] bf16 rows, SWIZZLE_128B; M -> 32x32 fp32.
    for (int idx = tid; idx < kCols * 8; idx += kThreads) {
        const int d = idx >> 3, ch = idx & 7;
        const int j0 = (ch & 3) * 8;
        const bool lo = ch >= 4;
        const float *qrow = p.Q + (size_t)(col0 + d) * r;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint16_t h2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = j0 + 2 * e + u;
                const float q = j < r ? __ldg(qrow + j) : 0.f;
                const uint16_t hi = bf16_bits(q);
                h2[u] = lo ? bf16_bits(q - bf16_val(hi)) : hi;
            }
            w[e] = uint32_t(h2[0]) | (uint32_t(h2[1]) << 16);
        }
        *reinterpret_cast<uint4 *>(sq + d * 128 + swz(d, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int idx = tid; idx < 32 * 32; idx += kThreads) {  // sm[k][j] = M[j][k]
        const int k = idx >> 5, j = idx & 31;
        sm[idx] = (j < r && k < r) ? __ldg(p.M + j * r + k) : 0.f;
    }
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    cluster_sync();  // barriers initialised in every CTA before any push
    // Q and M are staged above while the previous kernel of the stream may still
    // run; x and every output only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    {
        const int quad = warp & 3, part = warp >> 2;
        const int m = quad * 32 + lane;  // tile row == TMEM lane
        const uint32_t lane_base = uint32_t(quad * 32) << 16;
        const uint32_t tcol = uint32_t(part * kPartCols);
        const uint32_t idesc_y = idesc_bf16_f32(128, 64, false, true);
        const uint32_t idesc_c = idesc_bf16_f32(128, 128, false, false);
        const uint32_t slab_tx = uint32_t(R * 128);
        if (tid == 0 && has_tile(0)) {
#pragma unroll 1
            for (int s = 0; s < kSlabs; ++s) {
                if (err) break;  // no arming without the load that completes it
                mbar_expect_tx(bar(kBarLd + s), slab_tx);
                tma_load_2d(smem_u32(sx + s * kSlabBytes), &tm_x, col0 + s * kSlabCols, int(tile_t0(0)),
                            bar(kBarLd + s));
            }
        }

        // INT3 codes (three 8-byte stores per 64 codes) are stored while the next
        // tile's first cluster barrier settles, so that its release does not wait
        // for them (measured: faster for INT3, slower for the single 32-byte INT4
        // store, which leaves at once)
        uint32_t pend[4 * (kQuant ? BITS : 1)];
        uint8_t *pend_dst = nullptr;
        auto store_pending = [&]() {
            if (pend_dst) {
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2) {
                    uint8_t *dst = pend_dst + b2 * (BITS * 8);
                    const uint32_t *w = pend + b2 * 2 * BITS;
                    if (BITS == 4 && p.codes_v8) {
                        st_global_v8(dst, w);
                    } else if (BITS == 4) {
                        reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    } else {
                        reinterpret_cast<uint2 *>(dst)[0] = make_uint2(w[0], w[1]);
                        reinterpret_cast<uint2 *>(dst)[1] = make_uint2(w[2], w[3]);
                        reinterpret_cast<uint2 *>(dst)[2] = make_uint2(w[4], w[5]);
                    }
                }
                pend_dst = nullptr;
            }
        };

        for (int it = 0; has_tile(it); ++it) {
            const uint32_t ph = uint32_t(it) & 1u;
            const long long t0 = tile_t0(it);
            const int nrows = int(p.T - t0 < R ? p.T - t0 : R);
            const bool next = has_tile(it + 1);

            // ---- y = x [Q_hi | Q_lo] over this CTA's 512 columns, slab by slab as the tile lands
            if (tid == 0) {
                const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(sx), 1024));
                const uint64_t bd0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
#pragma unroll 1
                for (int s = 0; s < kSlabs; ++s) {
                    if (!mbar_wait(bar(kBarLd + s), ph, err != 0)) err |= kErrMbarTimeout;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // K steps of 16 columns, 32 bytes apart
                        const int i = 4 * s + k;
                        const uint32_t aoff = uint32_t(s * kSlabBytes + k * 32) >> 4;
                        const uint32_t boff = uint32_t(i * 2048) >> 4;
                        if (!err) umma_f16(tmem, ad0 + aoff, bd0 + boff, idesc_y, i != 0);
                    }
                }
                if (!err) umma_commit(bar(kBarY));
                if (next) {  // the next tile into L2 while this one is processed
                    const int tn = int(tile_t0(it + 1));
#pragma unroll 1
                    for (int s = 0; s < kSlabs; ++s) tma_prefetch_2d(&tm_x, col0 + s * kSlabCols, tn);
                }
            }
            __syncwarp();  // lanes of warp 0 wait here, not in a poll that competes with lane 0

            // ---- partial projection of this CTA's columns -> operand buffer (fp32)
            if (part == 0) {
                if (!mbar_wait(bar(kBarY), ph, err != 0)) err |= kErrMbarTimeout;
                tc_fence_after();
                uint32_t a[32], b[32];
                tmem_ld32(tmem + lane_base + 0, a);
                tmem_ld32(tmem + lane_base + 32, b);
                tmem_wait_ld();
                uint8_t *prow = sz + m * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float4 v;
                    v.x = __uint_as_float(a[4 * c + 0]) + __uint_as_float(b[4 * c + 0]);
                    v.y = __uint_as_float(a[4 * c + 1]) + __uint_as_float(b[4 * c + 1]);
                    v.z = __uint_as_float(a[4 * c + 2]) + __uint_as_float(b[4 * c + 2]);
                    v.w = __uint_as_float(a[4 * c + 3]) + __uint_as_float(b[4 * c + 3]);
                    *reinterpret_cast<float4 *>(prow + swz(m, c)) = v;
                }
            }
            tc_fence_before();
            cluster_arrive();  // #1 partial projections of all CTAs are visible
            store_pending();
            cluster_wait();

            // ---- owner CTA: sum the partials of its TPO rows (one warp per row, one
            // projection entry per lane), z = M y, push z hi|lo to every CTA
            if (warp < TPO) {
                const int kq = lane;
                const int mo = int(crank) * TPO + warp;
                const uint32_t row_addr = smem_u32(sz + mo * 128);
                float pv[CS];
#pragma unroll
                for (int c = 0; c < CS; ++c)
                    pv[c] = ld_dsmem_f32(mapa(row_addr, uint32_t(c)) + swz(mo, kq >> 2) + 4 * (kq & 3));
                float y = 0.f;
#pragma unroll
                for (int c = 0; c < CS; ++c) y += pv[c];
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) acc = fmaf(sm[k * 32 + kq], __shfl_sync(0xFFFFFFFFu, y, k), acc);
                const uint16_t hi = bf16_bits(acc), lo = bf16_bits(acc - bf16_val(hi));
                const uint32_t hl = uint32_t(hi) | (uint32_t(lo) << 16);
                // lane -> 16-byte chunk ch of the row (hi: z[8 ch ..], lo: z[8 (ch - 4) ..])
                const int ch = lane & 7;
                const int src0 = 8 * (ch & 3);
                const int sh = ch >= 4 ? 16 : 0;
                uint32_t hw[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) hw[e] = (__shfl_sync(0xFFFFFFFFu, hl, src0 + e) >> sh) & 0xFFFFu;
                const uint32_t w0 = hw[0] | (hw[1] << 16), w1 = hw[2] | (hw[3] << 16);
                const uint32_t w2 = hw[4] | (hw[5] << 16), w3 = hw[6] | (hw[7] << 16);
                // the row goes into this CTA's operand buffer (its own partial has been
                // read above), then by bulk copy (async proxy, like the tensor core that
                // reads it) into the same row of every other CTA
                if (lane < 8) *reinterpret_cast<uint4 *>(sz + mo * 128 + swz(mo, ch)) = make_uint4(w0, w1, w2, w3);
                fence_proxy_async_cta();
                __syncwarp();
                if (lane < CS && lane != int(crank))
                    if (!err) bulk_copy_to_cluster(mapa(row_addr, uint32_t(lane)), row_addr, 128u,
                                         mapa(bar(kBarZ), uint32_t(lane)));
                if (lane == 0 && !err) mbar_arrive(bar(kBarZ));
            }

            // ---- c = z Q^T (hi/lo split): quarter q into TMEM columns [128 q, 128 q + 128),
            // in column-part order, issued by a warp of the last part (whose quarter lands
            // last anyway), so that parts 0-2 start pass 1 as soon as theirs is done
            if (warp == kMma2Warp && lane == 0) {
                if (!mbar_wait(bar(kBarZ), ph, err != 0)) err |= kErrMbarTimeout;
                if (next && !err) mbar_expect_tx(bar(kBarZ), uint32_t(kZTx));
                tc_fence_after();
                fence_proxy_async();
                const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(sz), 1024));
                const uint64_t bd0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
                // (A K-step, B K-step) pairs: z_hi Q_hi^T, z_hi Q_lo^T, z_lo Q_hi^T
                constexpr uint32_t kA[6] = {0, 1, 0, 1, 2, 3}, kB[6] = {0, 1, 2, 3, 0, 1};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
#pragma unroll
                    for (int s = 0; s < 6; ++s)
                        if (!err) umma_f16(tmem + q * 128, ad0 + ((kA[s] * 32) >> 4),
                                 bd0 + ((uint32_t(q) * 16384 + kB[s] * 32) >> 4), idesc_c, s != 0);
                    if (!err) umma_commit(bar(kBarC + q));
                }
            }
            __syncwarp();

            // ---- pass 1: x_out = x + c over this warp's 128 columns (TMEM loads pipelined:
            // the load of the next 32-column block overlaps the arithmetic of the current one)
            if (!mbar_wait(bar(kBarLd + 2 * part), ph, err != 0)) err |= kErrMbarTimeout;
            if (!mbar_wait(bar(kBarLd + 2 * part + 1), ph, err != 0)) err |= kErrMbarTimeout;
            if (!mbar_wait(bar(kBarC + part), ph, err != 0)) err |= kErrMbarTimeout;
            tc_fence_after();
            double ss = 0.0;
            float amax = 0.f;
            {
                float2 s2 = make_float2(0.f, 0.f);
                float am[4] = {0.f, 0.f, 0.f, 0.f};
                constexpr int kBlocks = kPartCols / 32;
                uint32_t va[32], vb[32];
                const uint32_t taddr = tmem + lane_base + tcol;
                uint8_t *xbase = sx + m * 128;
                tmem_ld32(taddr, va);
                tmem_wait_ld();
#pragma unroll 1
                for (int b = 0; b < kBlocks; b += 2) {
                    const int cb = part * kBlocks + b;  // 32-column block within the CTA slice
                    tmem_wait_st();
                    tmem_ld32(taddr + (b + 1) * 32, vb);
                    xout_block(va, xbase + (cb >> 1) * kSlabBytes, m, (cb & 1) * 4, s2, am);
                    if (kQuant) tmem_st32(taddr + b * 32, va);  // fp32 x_out for the codes
                    tmem_wait_ld();
                    tmem_wait_st();
                    if (b + 2 < kBlocks) tmem_ld32(taddr + (b + 2) * 32, va);
                    xout_block(vb, xbase + ((cb + 1) >> 1) * kSlabBytes, m, ((cb + 1) & 1) * 4, s2, am);
                    if (kQuant) tmem_st32(taddr + (b + 1) * 32, vb);
                    tmem_wait_ld();
                    // fold the fp32 pair sums of these 64 columns into float64
                    ss += double(s2.x) + double(s2.y);
                    s2 = make_float2(0.f, 0.f);
                }
                tmem_wait_st();
                amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
            }
            fence_proxy_async_cta();  // x_out (generic writes) -> TMA store (async proxy)
            // statistics: fold the column parts of each row; part 0 pushes the CTA's
            // partial (ss, amax) of row m to the row's owner
            if (kQuant && part > 0) {
                reinterpret_cast<double *>(sloc + ((part - 1) * kTileM + m) * 16)[0] = ss;
                reinterpret_cast<float *>(sloc + ((part - 1) * kTileM + m) * 16)[2] = amax;
            }
            named_sync(1, kConsumers);
            if (warp == kConsumerWarps - 1) {
                // x_out back to HBM, one bulk group per slab; each slab takes the next
                // tile as soon as its store has read it (a warp with no statistics
                // duty; the whole warp waits for its lane 0)
                if (lane == 0) {
#pragma unroll 1
                    for (int s = 0; s < kSlabs; ++s) {
                        if (!err) tma_store_2d(&tm_xo, smem_u32(sx + s * kSlabBytes), col0 + s * kSlabCols, int(t0));
                        bulk_commit();
                    }
                    if (next) {
                        const int tn = int(tile_t0(it + 1));
#pragma unroll 1
                        for (int s = 0; s < kSlabs; ++s) {
                            bulk_wait_read_n(kSlabs - 1 - s);
                            if (err) break;  // no arming without the load that completes it
                            mbar_expect_tx(bar(kBarLd + s), slab_tx);
                            tma_load_2d(smem_u32(sx + s * kSlabBytes), &tm_x, col0 + s * kSlabCols, tn,
                                        bar(kBarLd + s));
                        }
                    }
                }
                __syncwarp();
            }
            if constexpr (kQuant) {
            if (part == 0) {
#pragma unroll
                for (int k = 0; k < kParts - 1; ++k) {
                    ss += reinterpret_cast<const double *>(sloc + (k * kTileM + m) * 16)[0];
                    amax = fmaxf(amax, reinterpret_cast<const float *>(sloc + (k * kTileM + m) * 16)[2]);
                }
                const uint32_t owner = uint32_t(m / TPO);
                const uint32_t dst = smem_u32(sst + (int(crank) * TPO + m % TPO) * 16);
                if (!err) st_async_v4(mapa(dst, owner), uint32_t(__double2loint(ss)), uint32_t(__double2hiint(ss)),
                            __float_as_uint(amax), 0u, mapa(bar(kBarSt), owner));
            }

            // ---- owner: totals of its rows over the cluster in a fixed order
            // (deterministic), scale, row quantiser pushed to every CTA
            constexpr int kStatThreads = TPO * CS;  // one per (own row, destination CTA)
            if (tid < kStatThreads) {
                const int rl = tid / CS, dst_cta = tid % CS;
                if (!mbar_wait(bar(kBarSt), ph, err != 0)) err |= kErrMbarTimeout;
                double ss_t = 0.0;
                float am_t = 0.f;
#pragma unroll
                for (int c = 0; c < CS; ++c) {
                    const float4 v = *reinterpret_cast<const float4 *>(sst + (c * TPO + rl) * 16);
                    ss_t += __hiloint2double(__float_as_int(v.y), __float_as_int(v.x));
                    am_t = fmaxf(am_t, v.z);
                }
                const int mo = int(crank) * TPO + rl;
                const float ms = float(ss_t / double(p.D));
                const float rs = 1.0f / sqrtf(ms + p.eps);
                const RowQuant q = row_quant(am_t, qmax);
                if (dst_cta == 0 && mo < nrows) p.scales[t0 + mo] = am_t > 0.f ? (am_t * rs) / float(qmax) : 0.f;
                if (!err) st_async_v2(mapa(smem_u32(sprm + mo * 8), uint32_t(dst_cta)), __float_as_uint(q.inv),
                            __float_as_uint(q.pre), mapa(bar(kBarPrm), uint32_t(dst_cta)));
                if (tid == 0 && next && !err) mbar_expect_tx(bar(kBarSt), uint32_t(CS * TPO * 16));
            }
            if (!mbar_wait(bar(kBarPrm), ph, err != 0)) err |= kErrMbarTimeout;
            if (tid == 0 && next && !err) mbar_expect_tx(bar(kBarPrm), uint32_t(kTileM * 8));
            RowQuant rq;
            rq.inv = reinterpret_cast<const float *>(sprm + m * 8)[0];
            rq.pre = reinterpret_cast<const float *>(sprm + m * 8)[1];
            const bool valid = m < nrows;

            // ---- pass 2: codes from the fp32 x_out in TMEM (loads pipelined)
            {
                constexpr int kBlocks = kPartCols / 32;
                const uint32_t taddr = tmem + lane_base + tcol;
                uint8_t *crow = p.codes + (t0 + m) * row_bytes + (long long)(col0 + part * kPartCols) * BITS / 8;
                uint32_t va[32], vb[32];
                tmem_ld32(taddr, va);
                tmem_wait_ld();
#pragma unroll
                for (int b = 0; b < kBlocks; b += 2) {
                    uint32_t *words = pend + (b / 2) * 2 * BITS;  // 64 codes
                    tmem_ld32(taddr + (b + 1) * 32, vb);
                    code_block<BITS>(va, rq, words);
                    tmem_wait_ld();
                    if (b + 2 < kBlocks) tmem_ld32(taddr + (b + 2) * 32, va);
                    code_block<BITS>(vb, rq, words + BITS);
                    if (BITS == 4 && valid) {
                        uint8_t *dst = crow + (b / 2) * (BITS * 8);
                        if (p.codes_v8) {
                            st_global_v8(dst, words);
                        } else {
                            reinterpret_cast<uint4 *>(dst)[0] = make_uint4(words[0], words[1], words[2], words[3]);
                            reinterpret_cast<uint4 *>(dst)[1] = make_uint4(words[4], words[5], words[6], words[7]);
                        }
                    }
                    tmem_wait_ld();
                }
                if (BITS == 3 && valid) pend_dst = crow;
            }
            }
            tc_fence_before();
            named_sync(1, kConsumers);  // TMEM reads done before the next tile's products
            tc_fence_after();
        }
        store_pending();
        if (warp == kConsumerWarps - 1 && lane == 0) bulk_wait0();
    }

    tc_fence_before();
    // after a failed wait no further asynchronous work was issued: let what was
    // already in flight land before TMEM is freed and the CTA exits
    if (__syncthreads_or(err)) drain_delay();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(p.status, err);
    cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

// -------------------------------------------------------------------- host
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

bool make_map(CUtensorMap *m, const void *ptr, long long T, int D, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kSlabCols), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CS, int BITS>
struct TcKernel {
    static int max_clusters[64];
    static bool configured[64];

    static cudaError_t configure(int dev) {
        if (configured[dev]) return cudaSuccess;
        auto kern = k_align_tc<CS, BITS>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<CS>::kSmem);
        if (e != cudaSuccess) return e;
        if (CS > 8) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
        }
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(CS, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = Layout<CS>::kSmem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return e;
        max_clusters[dev] = n;
        configured[dev] = true;
        return cudaSuccess;
    }

    static cudaError_t launch(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                              float *scales, long long T, int D, int r, float eps, int *status, cudaStream_t s,
                              bool *launched) {
        *launched = false;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaSuccess;
        e = configure(dev);
        if (e != cudaSuccess) return e;
        const int maxcl = max_clusters[dev];
        if (maxcl < 1) return cudaSuccess;  // cannot co-schedule this cluster shape: caller uses another kernel
        const long long base_tiles = (T + kTileM - 1) / kTileM;
        const int ncl = int(base_tiles < maxcl ? base_tiles : maxcl);
        const int tpc = int((base_tiles + ncl - 1) / ncl);
        const long long ntiles = (long long)ncl * tpc;
        const int R = int((T + ntiles - 1) / ntiles);
        CUtensorMap mx, mxo;
        if (!make_map(&mx, x, T, D, R) || !make_map(&mxo, x_out, T, D, R)) return cudaErrorInvalidValue;
        AlignTcArgs a;
        a.Q = Q;
        a.M = M;
        a.codes = codes;
        a.scales = scales;
        a.status = status;
        a.T = T;
        a.D = D;
        a.r = r;
        a.rows_per_tile = R;
        a.tiles_per_cluster = tpc;
        a.codes_v8 = (reinterpret_cast<uintptr_t>(codes) & 31u) == 0;
        a.eps = eps;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3(CS * ncl, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = Layout<CS>::kSmem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_align_tc<CS, BITS>, mx, mxo, a);
        if (e == cudaSuccess) {
            *launched = true;
            count_launch();
        }
        return e;
    }
};

template <int CS, int BITS>
int TcKernel<CS, BITS>::max_clusters[64];
template <int CS, int BITS>
bool TcKernel<CS, BITS>::configured[64];

}  // namespace

bool align_tc_supports(int D, int r, int dtype, long long T) {
    return dtype == 1 && (D == 4096 || D == 8192) && r >= 1 && r <= 32 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_align_tc(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                            float *scales, long long T, int D, int r, int bits, float eps, cudaStream_t s,
                            bool *launched) {
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    if (D == 4096) {
        if (bits == 0) return TcKernel<8, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
        return bits == 4 ? TcKernel<8, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched)
                         : TcKernel<8, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    }
    if (bits == 0) return TcKernel<16, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    return bits == 4 ? TcKernel<16, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched)
                     : TcKernel<16, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
}

}  // namespace rsq
