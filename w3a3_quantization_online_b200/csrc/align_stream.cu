// align_stream.cu -- tensor-core residual subspace alignment fused with the
// weight-free RMSNorm and the per-token symmetric quantiser, bf16 I/O,
// D in {4096, 8192}: clusters of D / 1024 CTAs, each token tile streamed three
// times through a small shared-memory ring (from HBM once, from L2 twice).
//
// ReSpinQuant paper notes, key design 3: y = Q^T x (D -> r), z = M y,
// x_out = x + Q z.  Infra Quant II, QuaRot / Method: scale-free RMSNorm in FP32
// and per-token symmetric absmax quantisation (SpinQuant / Motivation gives
// alpha = max|X| / (2^(N-1) - 1)).
//
// Design (B200, sm_100a):
//  * CTA c of a cluster owns hidden columns [1024 c, 1024 c + 1024) and keeps
//    its 1024 x 32 slice of Q resident in shared memory as bf16 [Q_hi | Q_lo]
//    (128 KB).  Clusters of 4 (D = 4096) co-schedule on 132 SMs.
//  * A token tile (R <= 128 rows) is never resident: its sixteen 64-column
//    slabs (16 KB each) stream through a 4-stage TMA ring three times.
//    Pass 0 (from HBM; the tile was prefetched into L2 while the previous tile
//    was processed) feeds the projection y = x [Q_hi | Q_lo] (M = 128, N = 64,
//    K = 1024) into TMEM columns 0-63.  Pass 1 (an L2 hit) gives the row
//    statistics of x_out = x + c, where c = z_hi Q_hi^T + z_hi Q_lo^T +
//    z_lo Q_hi^T is formed per 256-column chunk (M = 128, N = 256, K = 96) into
//    one of two TMEM buffers.  Pass 2 (L2 again) forms the same c again, writes
//    bf16 x_out in place over the slab (stored by TMA) and the codes from the
//    fp32 x_out.  x_out is written only in pass 2, so x_out may be x.
//  * Warp 8 issues the TMA loads, warp 9 the tensor-core products, warp 10 the
//    x_out stores and the release of every slab the epilogue reads.  Warps 0-7
//    are the epilogue: two per TMEM lane quadrant (one token row per thread),
//    warps 0-3 on the even slabs, warps 4-7 on the odd ones, so each half owns
//    two stages of the ring.
//  * Exchanges, each a push counted on an mbarrier of the receiving CTA:
//    partial projections (fp32, st.async) to the rows' owner CTA, which sums
//    them in a fixed order, forms z = M y, writes its rows of z (bf16 hi|lo)
//    into its own operand buffer and copies them (one bulk copy per CTA) into
//    every other CTA's; row statistics (st.async) to the owner, which forms the
//    scale and the row quantiser and pushes the quantiser to every CTA.
//    Every exchange needs every CTA of the cluster, so no CTA runs a whole
//    tile ahead of another and one buffer per exchange suffices.
//  * Programmatic dependent launch: Q and M are staged before the wait on the
//    previous kernel of the stream; x and every output only after it.
// Every mbarrier wait is bounded (2 s of %globaltimer).  A timeout sets a bit in
// the device status word; after a failed wait a thread issues no further
// asynchronous work and returns from every later wait at once, and the CTA
// drains what is in flight before freeing TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kTileM = 128;                  // token rows per tile (MMA M)
constexpr int kCols = 1024;                  // hidden columns owned by one CTA
constexpr int kSlabCols = 64;                // bf16 columns per 128-byte swizzle row
constexpr int kSlabs = kCols / kSlabCols;    // 16 per pass
constexpr int kChunkCols = 256;              // columns of c per product (N)
constexpr int kChunks = kCols / kChunkCols;  // 4 per pass
constexpr int kSlabBytes = kTileM * 128;     // 16 KB
constexpr int kStages = 4;                   // two per epilogue half
constexpr int kQBytes = kCols * 128;         // 128 KB: [Q_hi(32) | Q_lo(32)] bf16 per row
constexpr int kZBytes = kTileM * 128;        // 16 KB: z hi|lo per row
constexpr int kEpiWarps = 8;
constexpr int kEpi = kEpiWarps * 32;
constexpr int kLoadWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1, kStoreWarp = kEpiWarps + 2;
constexpr int kThreads = kEpi + 96;
constexpr int kTmemCols = 512;
static_assert(kSlabs % kStages == 0 && kStages % 2 == 0, "ring stages split evenly between the halves");
static_assert(kChunkCols == 4 * kSlabCols, "a chunk is four slabs, two per half");

struct StreamArgs {
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
    int codes_v8;
    float eps;
};

enum : int {
    kBarFull = 0,                     // [4] slab landed (TMA)
    kBarEmpty = kBarFull + kStages,   // [4] slab free for the next load
    kBarReady = kBarEmpty + kStages,  // [4] slab read (pass 1) or x_out written (pass 2) by its half
    kBarY = kBarReady + kStages,      // projection of the tile done (commit)
    kBarRy,                           // owner: partial projections of its rows from every CTA
    kBarZ,                            // z of every row in the operand buffer
    kBarC,                            // [2] c of a chunk in TMEM buffer b (commit)
    kBarTF = kBarC + 2,               // [2] TMEM buffer b read by the epilogue
    kBarSt = kBarTF + 2,              // owner: row statistics from every CTA
    kBarPrm,                          // row quantisers of the tile
    kNumBars
};

template <int CS>
struct StreamLayout {
    static constexpr int TPO = kTileM / CS;                  // rows owned per CTA per tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffX = kOffQ + kQBytes;            // [4] slab ring
    static constexpr int kOffZ = kOffX + kStages * kSlabBytes;
    // owner: [CS source][TPO rows][32] fp32 partial projections.  Later in the
    // tile the same bytes hold the row statistics received from every CTA
    // ([CS][TPO] x 16 B) and the second half's statistics of each row
    // ([128] x 16 B): no CTA sends the next tile's partials before it has the
    // quantisers of every row, which the owners send after reading both.
    static constexpr int kOffR = kOffZ + kZBytes;
    static constexpr int kOffSt = kOffR;
    static constexpr int kOffScr = kOffR + CS * TPO * 16;
    static constexpr int kOffPrm = kOffR + CS * TPO * 128;   // [128 rows] (inv, pre)
    static constexpr int kOffBar = kOffPrm + kTileM * 8;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;  // TMEM address, then [CS + 1] error flags
    static constexpr int kBytes = kOffTmem + 48;
    static constexpr int kSmem = kBytes + 1024;
    static_assert(kOffX % 1024 == 0 && kOffZ % 1024 == 0, "swizzle atoms");
    static_assert(kOffScr + kTileM * 16 <= kOffPrm, "statistics fit in the partials buffer");
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return uint32_t(((chunk ^ (row & 7)) << 4)); }

__device__ __forceinline__ uint64_t opaque(uint64_t v) {
    asm volatile("mov.b64 %0, %0;" : "+l"(v));
    return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t *>(&h);
}

__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

// x_out = x + c on 32 columns of row m: v holds c on entry and fp32 x_out on
// return; x from the 16-byte chunks chunk0 .. chunk0 + 3 of the swizzled slab
// row.  STATS: sums of squares in pairs and four partial maxima; STORE: the
// bf16 x_out goes back over x.
template <bool STATS, bool STORE>
__device__ __forceinline__ void xout_block(uint32_t (&v)[32], uint8_t *srow, int m, int chunk0, float2 &s2,
                                           float (&am)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 *p = reinterpret_cast<uint4 *>(srow + swz(m, chunk0 + c));
        const uint4 xw = *p;
        const uint32_t xs[4] = {xw.x, xw.y, xw.z, xw.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x2 = make_float2(__uint_as_float(xs[e] << 16), __uint_as_float(xs[e] & 0xFFFF0000u));
            const float2 c2 = make_float2(__uint_as_float(v[c * 8 + 2 * e]), __uint_as_float(v[c * 8 + 2 * e + 1]));
            const float2 y = add2(x2, c2);
            v[c * 8 + 2 * e] = __float_as_uint(y.x);
            v[c * 8 + 2 * e + 1] = __float_as_uint(y.y);
            if (STATS) {
                s2 = fma2(y, y, s2);
                am[e] = max3(am[e], fabsf(y.x), fabsf(y.y));
            }
            if (STORE) o[e] = pack_bf16x2(y.x, y.y);
        }
        if (STORE) *p = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Codes of 32 fp32 values: BITS words.
template <int BITS>
__device__ __forceinline__ void code_block(const uint32_t (&v)[32], const RowQuant &rq, uint32_t *words) {
    uint32_t g[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[gi * 8 + e]);
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
k_align_stream(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xo,
               const StreamArgs p) {
    using L = StreamLayout<CS>;
    constexpr int TPO = L::TPO;
    constexpr bool kQuant = BITS > 0;
    constexpr int kPasses = kQuant ? 3 : 2;  // slab passes per tile (no statistics pass without codes)
    constexpr uint32_t kRyTx = uint32_t(CS * TPO * 128);
    constexpr uint32_t kZTx = uint32_t((CS - 1) * TPO * 128);
    constexpr uint32_t kStTx = uint32_t(CS * TPO * 16);
    constexpr uint32_t kPrmTx = uint32_t(kTileM * 8);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = base + L::kOffQ;
    uint8_t *sz = base + L::kOffZ;
    float *srecv = reinterpret_cast<float *>(base + L::kOffR);
    uint8_t *sst = base + L::kOffSt;
    uint8_t *sscr = base + L::kOffScr;
    uint8_t *sprm = base + L::kOffPrm;
    auto slab = [&](int st) { return base + L::kOffX + st * kSlabBytes; };
    const uint32_t bars = smem_u32(base + L::kOffBar);
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L::kOffTmem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
    const int col0 = int(crank) * kCols;
    const int r = p.r;
    const int qmax = kQuant ? (1 << (BITS - 1)) - 1 : 1;
    const long long row_bytes = (long long)p.D * (kQuant ? BITS : 4) / 8;
    const int R = p.rows_per_tile;
    int err = 0;
    auto wait = [&](int b, uint32_t ph) {
        if (!mbar_wait(bar(b), ph, err != 0)) err |= kErrMbarTimeout;
    };

    asm volatile("griddepcontrol.launch_dependents;");
    auto tile_t0 = [&](int it) { return ((long long)cid + (long long)it * ncl) * R; };
    int nt = 0;
    while (nt < p.tiles_per_cluster && tile_t0(nt) < p.T) ++nt;
    // ring position of slab s of pass ps (0 projection, 1 statistics, 2 output)
    // of tile it, and its ordinal among the slabs the epilogue reads
    auto pidx = [&](int ps) { return kQuant ? ps : (ps == 0 ? 0 : 1); };
    auto seq = [&](int it, int ps, int s) { return (it * kPasses + pidx(ps)) * kSlabs + s; };
    auto epi_seq = [&](int it, int ps, int s) { return (it * (kPasses - 1) + pidx(ps) - 1) * kSlabs + s; };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i >= kBarReady && i < kBarReady + kStages) cnt = 4;  // the four warps of a half
            if (i == kBarZ) cnt = 1 + kEpiWarps;
            if (i == kBarTF || i == kBarTF + 1) cnt = kEpiWarps;
            mbar_init(bar(i), cnt);
        }
        fence_mbar_init();
        if (nt > 0) {
            mbar_expect_tx(bar(kBarRy), kRyTx);
            mbar_expect_tx(bar(kBarZ), kZTx);
            if (kQuant) {
                mbar_expect_tx(bar(kBarSt), kStTx);
                mbar_expect_tx(bar(kBarPrm), kPrmTx);
            }
        }
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (tid == kLoadWarp * 32) prefetch_tmap(&tm_x);
    if (tid == kStoreWarp * 32) prefetch_tmap(&tm_xo);
    // Q slice -> [Q_hi | Q_lo] bf16 rows (SWIZZLE_128B): one row serves as the
    // MN-major B operand of the projection and the K-major B operand of c
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
                const float qv = j < r ? __ldg(qrow + j) : 0.f;
                const uint16_t hi = bf16_bits(qv);
                h2[u] = lo ? bf16_bits(qv - bf16_val(hi)) : hi;
            }
            w[e] = uint32_t(h2[0]) | (uint32_t(h2[1]) << 16);
        }
        *reinterpret_cast<uint4 *>(sq + d * 128 + swz(d, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    // row `lane` of M in registers (the owner step's z = M y)
    float mrow[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) mrow[k] = (warp < kEpiWarps && lane < r && k < r) ? __ldg(p.M + lane * r + k) : 0.f;
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    cluster_sync();  // barriers initialised in every CTA before any push
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const uint32_t slab_tx = uint32_t(R * 128);

    if (warp == kLoadWarp) {
        // ======================= TMA loads: three passes over each tile's slabs
        if (lane == 0) {
#pragma unroll 1
            for (int it = 0; it < nt; ++it) {
                const int t0 = int(tile_t0(it));
#pragma unroll 1
                for (int ps = 0; ps < 3; ++ps) {
                    if (!kQuant && ps == 1) continue;
                    if (ps == 1 || (!kQuant && ps == 2)) {
                        // the next tile into L2 while this one is processed
                        if (it + 1 < nt && !err) {
                            const int tn = int(tile_t0(it + 1));
#pragma unroll 1
                            for (int s = 0; s < kSlabs; ++s) tma_prefetch_2d(&tm_x, col0 + s * kSlabCols, tn);
                        }
                    }
#pragma unroll 1
                    for (int s = 0; s < kSlabs; ++s) {
                        const int j = seq(it, ps, s), st = j % kStages;
                        if (j >= kStages) wait(kBarEmpty + st, uint32_t(j / kStages - 1) & 1u);
                        if (err) break;  // no arming without the load that completes it
                        mbar_expect_tx(bar(kBarFull + st), slab_tx);
                        tma_load_2d(smem_u32(slab(st)), &tm_x, col0 + s * kSlabCols, t0, bar(kBarFull + st));
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ======================= tensor-core products
        if (lane == 0) {
            const uint32_t idesc_y = idesc_bf16_f32(128, 64, false, true);
            const uint32_t idesc_c = idesc_bf16_f32(128, kChunkCols, false, false);
            // (A K-step, B K-step) pairs of c: z_hi Q_hi^T, z_hi Q_lo^T, z_lo Q_hi^T
            constexpr uint32_t kA[6] = {0, 1, 0, 1, 2, 3}, kB[6] = {0, 1, 2, 3, 0, 1};
            const uint64_t bq0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
            const uint64_t az = opaque(smem_desc_sw128(smem_u32(sz), 1024));
            int uses[2] = {0, 0};  // products issued into each TMEM buffer so far
            auto free_buffer = [&](int b) {
                if (uses[b] > 0) wait(kBarTF + b, uint32_t(uses[b] - 1) & 1u);
            };
#pragma unroll 1
            for (int it = 0; it < nt; ++it) {
                // projection into columns 0-63 (inside buffer 0), slab by slab as pass 0 lands.
                // Both buffers released: the previous tile's last chunk has been read, so
                // its last pass-2 slabs have landed in the stages this tile's first slabs
                // reuse, and a parity wait on those stages' full barriers is exact (without
                // it the wait could match the older phase and release a stage twice).
                free_buffer(0);
                free_buffer(1);
                tc_fence_after();
#pragma unroll 1
                for (int s = 0; s < kSlabs; ++s) {
                    const int j = seq(it, 0, s), st = j % kStages;
                    wait(kBarFull + st, uint32_t(j / kStages) & 1u);
                    tc_fence_after();
                    const uint64_t ad = opaque(smem_desc_sw128(smem_u32(slab(st)), 1024));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // K steps of 16 columns, 32 bytes apart
                        const int i = 4 * s + k;
                        if (!err) umma_f16(tmem, ad + (uint32_t(k * 32) >> 4), bq0 + (uint32_t(i * 2048) >> 4), idesc_y,
                                           i != 0);
                    }
                    if (!err) umma_commit(bar(kBarEmpty + st));  // the slab may take its next load
                }
                if (!err) umma_commit(bar(kBarY));
                // z of every row present: c chunk by chunk, for pass 1 and again for pass 2
                wait(kBarZ, uint32_t(it) & 1u);
                if (it + 1 < nt && !err) mbar_expect_tx(bar(kBarZ), kZTx);
                tc_fence_after();
                fence_proxy_async();
#pragma unroll 1
                for (int ps = kQuant ? 1 : 2; ps <= 2; ++ps) {
#pragma unroll 1
                    for (int c = 0; c < kChunks; ++c) {
                        const int b = c & 1;
                        free_buffer(b);
                        tc_fence_after();
#pragma unroll
                        for (int s = 0; s < 6; ++s)
                            if (!err) umma_f16(tmem + uint32_t(kChunkCols * b), az + ((kA[s] * 32) >> 4),
                                               bq0 + ((uint32_t(c) * (kChunkCols * 128) + kB[s] * 32) >> 4), idesc_c,
                                               s != 0);
                        if (!err) umma_commit(bar(kBarC + b));
                        ++uses[b];
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kStoreWarp) {
        // ======================= x_out stores; every slab the epilogue reads is released here
        if (lane == 0) {
#pragma unroll 1
            for (int it = 0; it < nt; ++it) {
                const int t0 = int(tile_t0(it));
#pragma unroll 1
                for (int ps = kQuant ? 1 : 2; ps <= 2; ++ps) {
#pragma unroll 1
                    for (int s = 0; s < kSlabs; ++s) {
                        const int st = seq(it, ps, s) % kStages;
                        wait(kBarReady + st, uint32_t(epi_seq(it, ps, s) / kStages) & 1u);
                        if (ps == 2) {
                            if (!err) tma_store_2d(&tm_xo, smem_u32(slab(st)), col0 + s * kSlabCols, t0);
                            bulk_commit();
                            bulk_wait_read0();  // the store has read the slab
                        }
                        if (!err) mbar_arrive(bar(kBarEmpty + st));
                    }
                }
            }
            bulk_wait0();
        }
        __syncwarp();
    } else {
        // ======================= epilogue: TMEM lane quadrant `quad`, slabs of parity `half`
        const int quad = warp & 3, half = warp >> 2;
        const int m = 32 * quad + lane;  // tile row == TMEM lane
        const uint32_t lane_base = uint32_t(32 * quad) << 16;
        int uses[2] = {0, 0};
#pragma unroll 1
        for (int it = 0; it < nt; ++it) {
            const uint32_t ph = uint32_t(it) & 1u;
            const long long t0 = tile_t0(it);
            const bool more = it + 1 < nt;

            // ---- partial projection of this CTA's columns -> the row's owner
            if (half == 0) {
                wait(kBarY, ph);
                __syncwarp();
                tc_fence_after();
                uint32_t a[32], b[32];
                tmem_ld32(tmem + lane_base + 0, a);
                tmem_ld32(tmem + lane_base + 32, b);
                tmem_wait_ld();
                tc_fence_before();
                const uint32_t owner = uint32_t(m / TPO);
                const uint32_t dst = mapa(smem_u32(srecv + (int(crank) * TPO + m % TPO) * 32), owner);
                const uint32_t mb = mapa(bar(kBarRy), owner);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = __float_as_uint(__uint_as_float(a[4 * c + e]) + __uint_as_float(b[4 * c + e]));
                    if (!err) st_async_v4(dst + 16u * c, w[0], w[1], w[2], w[3], mb);
                }
            }

            // ---- owner: its TPO rows (TPO / 8 per warp, one projection entry per
            // lane): sum the CS partials in a fixed order, z = M y, z hi|lo into
            // this CTA's operand buffer, then by bulk copy into every other CTA's
            wait(kBarRy, ph);
            if (tid == 0 && more && !err) mbar_expect_tx(bar(kBarRy), kRyTx);
#pragma unroll 1
            for (int rl = warp; rl < TPO; rl += kEpiWarps) {
                const int mo = int(crank) * TPO + rl;
                float y = 0.f;
#pragma unroll
                for (int c = 0; c < CS; ++c) y += srecv[(c * TPO + rl) * 32 + lane];
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) acc = fmaf(mrow[k], __shfl_sync(0xFFFFFFFFu, y, k), acc);
                const uint16_t hi = bf16_bits(acc), lo = bf16_bits(acc - bf16_val(hi));
                const uint32_t hl = uint32_t(hi) | (uint32_t(lo) << 16);
                // lane -> 16-byte chunk ch of the row (hi: z[8 ch ..], lo: z[8 (ch - 4) ..])
                const int ch = lane & 7, src0 = 8 * (ch & 3), sh = ch >= 4 ? 16 : 0;
                uint32_t hw[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) hw[e] = (__shfl_sync(0xFFFFFFFFu, hl, src0 + e) >> sh) & 0xFFFFu;
                if (lane < 8)
                    *reinterpret_cast<uint4 *>(sz + mo * 128 + swz(mo, ch)) =
                        make_uint4(hw[0] | (hw[1] << 16), hw[2] | (hw[3] << 16), hw[4] | (hw[5] << 16),
                                   hw[6] | (hw[7] << 16));
            }
            fence_proxy_async_cta();  // z rows (generic writes) -> bulk copies and products (async proxy)
            named_sync(1, kEpi);
            if (tid == 0 && !err) {
                const uint32_t rows = smem_u32(sz + int(crank) * TPO * 128);
#pragma unroll 1
                for (int o = 0; o < CS; ++o)
                    if (o != int(crank))
                        bulk_copy_to_cluster(mapa(rows, uint32_t(o)), rows, uint32_t(TPO * 128),
                                             mapa(bar(kBarZ), uint32_t(o)));
            }
            __syncwarp();
            if (lane == 0 && !err) mbar_arrive(bar(kBarZ));

            // ---- pass 1: statistics of x_out = x + c (nothing is stored)
            RowQuant rq{1.f, 1.f};
            if constexpr (kQuant) {
                double ss = 0.0;
                float am[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
                for (int c = 0; c < kChunks; ++c) {
                    const int b = c & 1;
                    wait(kBarC + b, uint32_t(uses[b]) & 1u);
                    __syncwarp();
                    tc_fence_after();
#pragma unroll 1
                    for (int q2 = 0; q2 < 2; ++q2) {
                        const int sl = 4 * c + 2 * q2 + half;
                        const int j = seq(it, 1, sl), st = j % kStages;
                        const uint32_t taddr = tmem + lane_base + uint32_t(kChunkCols * b + kSlabCols * (2 * q2 + half));
                        uint32_t v0[32], v1[32];
                        tmem_ld32(taddr, v0);
                        tmem_ld32(taddr + 32, v1);
                        wait(kBarFull + st, uint32_t(j / kStages) & 1u);
                        __syncwarp();
                        tmem_wait_ld();
                        uint8_t *srow = slab(st) + m * 128;
                        float2 s2 = make_float2(0.f, 0.f);
                        xout_block<true, false>(v0, srow, m, 0, s2, am);
                        xout_block<true, false>(v1, srow, m, 4, s2, am);
                        ss += double(s2.x) + double(s2.y);
                        __syncwarp();
                        if (lane == 0 && !err) mbar_arrive(bar(kBarReady + st));
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0 && !err) mbar_arrive(bar(kBarTF + b));
                    ++uses[b];
                }
                float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));

                // ---- statistics: fold the halves, push the CTA's partial to the row's owner
                if (half == 1) {
                    reinterpret_cast<double *>(sscr + m * 16)[0] = ss;
                    reinterpret_cast<float *>(sscr + m * 16)[2] = amax;
                }
                named_sync(1, kEpi);
                if (half == 0) {
                    ss += reinterpret_cast<const double *>(sscr + m * 16)[0];
                    amax = fmaxf(amax, reinterpret_cast<const float *>(sscr + m * 16)[2]);
                    const uint32_t owner = uint32_t(m / TPO);
                    const uint32_t dst = smem_u32(sst + (int(crank) * TPO + m % TPO) * 16);
                    if (!err) st_async_v4(mapa(dst, owner), uint32_t(__double2loint(ss)), uint32_t(__double2hiint(ss)),
                                          __float_as_uint(amax), 0u, mapa(bar(kBarSt), owner));
                }
                // ---- owner: totals over the cluster in a fixed order (deterministic),
                // scale, row quantiser pushed to every CTA
                if (tid < CS * TPO) {
                    const int rl = tid / CS, dst_cta = tid % CS;
                    wait(kBarSt, ph);
                    if (tid == 0 && more && !err) mbar_expect_tx(bar(kBarSt), kStTx);
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
                    if (dst_cta == 0 && mo < R && t0 + mo < p.T)
                        p.scales[t0 + mo] = am_t > 0.f ? (am_t * rs) / float(qmax) : 0.f;
                    if (!err) st_async_v2(mapa(smem_u32(sprm + mo * 8), uint32_t(dst_cta)), __float_as_uint(q.inv),
                                          __float_as_uint(q.pre), mapa(bar(kBarPrm), uint32_t(dst_cta)));
                }
                wait(kBarPrm, ph);
                if (tid == 0 && more && !err) mbar_expect_tx(bar(kBarPrm), kPrmTx);
                rq.inv = reinterpret_cast<const float *>(sprm + m * 8)[0];
                rq.pre = reinterpret_cast<const float *>(sprm + m * 8)[1];
            }
            const bool valid = m < R && t0 + m < p.T;

            // ---- pass 2: bf16 x_out over the slab (stored by the store warp), codes of fp32 x_out
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
                const int b = c & 1;
                wait(kBarC + b, uint32_t(uses[b]) & 1u);
                __syncwarp();
                tc_fence_after();
#pragma unroll 1
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int sl = 4 * c + 2 * q2 + half;
                    const int j = seq(it, 2, sl), st = j % kStages;
                    const uint32_t taddr = tmem + lane_base + uint32_t(kChunkCols * b + kSlabCols * (2 * q2 + half));
                    uint32_t v0[32], v1[32];
                    tmem_ld32(taddr, v0);
                    tmem_ld32(taddr + 32, v1);
                    wait(kBarFull + st, uint32_t(j / kStages) & 1u);
                    __syncwarp();
                    tmem_wait_ld();
                    uint8_t *srow = slab(st) + m * 128;
                    float2 s2 = make_float2(0.f, 0.f);
                    float amd[4] = {0.f, 0.f, 0.f, 0.f};
                    xout_block<false, true>(v0, srow, m, 0, s2, amd);
                    xout_block<false, true>(v1, srow, m, 4, s2, amd);
                    fence_proxy_async_cta();  // bf16 x_out (generic writes) -> TMA store (async proxy)
                    __syncwarp();
                    if (lane == 0 && !err) mbar_arrive(bar(kBarReady + st));
                    if constexpr (kQuant) {
                        uint32_t words[2 * BITS];
                        code_block<BITS>(v0, rq, words);
                        code_block<BITS>(v1, rq, words + BITS);
                        if (valid) {
                            uint8_t *dst = p.codes + (t0 + m) * row_bytes + (long long)(col0 + kSlabCols * sl) * BITS / 8;
                            if (BITS == 4) {
                                if (p.codes_v8) {
                                    st_global_v8(dst, words);
                                } else {
                                    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(words[0], words[1], words[2], words[3]);
                                    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(words[4], words[5], words[6], words[7]);
                                }
                            } else {
                                reinterpret_cast<uint2 *>(dst)[0] = make_uint2(words[0], words[1]);
                                reinterpret_cast<uint2 *>(dst)[1] = make_uint2(words[2], words[3]);
                                reinterpret_cast<uint2 *>(dst)[2] = make_uint2(words[4], words[5]);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !err) mbar_arrive(bar(kBarTF + b));
                ++uses[b];
            }
        }
    }

    // Teardown.  After a failed wait a thread issues no further asynchronous work
    // and no mbarrier operation.  A peer may still have pushed into a CTA that
    // gave up waiting, so the CTAs first agree (through rank 0's shared memory)
    // whether any of them failed; if so every CTA lets what is in flight land
    // before TMEM is freed, and no CTA leaves before the last cluster barrier.
    tc_fence_before();
    const int cta_err = __syncthreads_or(err);
    uint32_t *flags = tmem_slot + 1;  // [CS], used in rank 0
    if (tid == 0) st_dsmem_u32(mapa(smem_u32(flags + crank), 0u), uint32_t(cta_err));
    cluster_sync();
    if (tid == 0) {
        uint32_t any = 0;
        for (int c = 0; c < CS; ++c) any |= uint32_t(ld_dsmem_u32(mapa(smem_u32(flags + c), 0u)));
        flags[CS] = any;
    }
    __syncthreads();
    if (flags[CS]) drain_delay();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(p.status, err);
    cluster_sync();  // no CTA leaves while a peer may still read or write its shared memory
}

// -------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// T x D bf16 row-major, boxes of 64 columns x box_rows rows, SWIZZLE_128B.
bool make_map(CUtensorMap *mp, const void *ptr, long long T, int D, int box_rows) {
    static EncodeTiledFn enc = nullptr;
    if (!enc) {
        void *q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) != cudaSuccess ||
            res != cudaDriverEntryPointSuccess)
            return false;
        enc = reinterpret_cast<EncodeTiledFn>(q);
    }
    const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kSlabCols), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CS, int BITS>
struct StreamKernel {
    static int max_clusters[64];
    static bool configured[64];

    static cudaLaunchAttribute cluster_attr() {
        cudaLaunchAttribute a = {};
        a.id = cudaLaunchAttributeClusterDimension;
        a.val.clusterDim.x = CS;
        a.val.clusterDim.y = 1;
        a.val.clusterDim.z = 1;
        return a;
    }

    static cudaError_t configure(int dev) {
        if (configured[dev]) return cudaSuccess;
        auto kern = k_align_stream<CS, BITS>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, StreamLayout<CS>::kSmem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1] = {cluster_attr()};
        cfg.gridDim = dim3(CS, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = StreamLayout<CS>::kSmem;
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
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaSuccess;
        e = configure(dev);
        if (e != cudaSuccess) return e;
        const int maxcl = max_clusters[dev];
        if (maxcl < 1) return cudaSuccess;
        // tiles of R <= 128 rows, the same number for every cluster
        const long long base_tiles = (T + kTileM - 1) / kTileM;
        const int ncl = int(base_tiles < maxcl ? base_tiles : maxcl);
        const int tpc = int((base_tiles + ncl - 1) / ncl);
        const long long ntiles = (long long)ncl * tpc;
        const int R = int((T + ntiles - 1) / ntiles);
        CUtensorMap mx, mxo;
        if (!make_map(&mx, x, T, D, R) || !make_map(&mxo, x_out, T, D, R)) return cudaErrorInvalidValue;
        StreamArgs a;
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
        cudaLaunchAttribute attr[2] = {cluster_attr(), cluster_attr()};
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3(CS * ncl, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = StreamLayout<CS>::kSmem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_align_stream<CS, BITS>, mx, mxo, a);
        if (e == cudaSuccess) {
            *launched = true;
            count_launch();
        }
        return e;
    }
};

template <int CS, int BITS>
int StreamKernel<CS, BITS>::max_clusters[64];
template <int CS, int BITS>
bool StreamKernel<CS, BITS>::configured[64];

}  // namespace

bool align_stream_supports(int D, int r, int dtype, long long T) {
    return dtype == 1 && (D == 4096 || D == 8192) && r >= 1 && r <= 32 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_align_stream(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                                float *scales, long long T, int D, int r, int bits, float eps, cudaStream_t s,
                                bool *launched) {
    *launched = false;
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    if (D == 4096) {
        if (bits == 0) return StreamKernel<4, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
        if (bits == 4) return StreamKernel<4, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
        return StreamKernel<4, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    }
    if (bits == 0) return StreamKernel<8, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    if (bits == 4) return StreamKernel<8, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    return StreamKernel<8, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
}

}  // namespace rsq
