// align_pipe.cu -- tensor-core residual subspace alignment fused with the
// weight-free RMSNorm and the per-token symmetric quantiser, bf16 I/O, with
// two 64-row tiles in flight per CTA.
//
// ReSpinQuant paper notes, key design 3: y = Q^T x (D -> r), z = M y,
// x_out = x + Q z.  Infra Quant II, QuaRot / Method: scale-free RMSNorm in FP32
// and per-token symmetric absmax quantisation (SpinQuant / Motivation gives
// alpha = max|X| / (2^(N-1) - 1)).
//
// Design (B200, sm_100a):
//  * A cluster of CS CTAs splits the hidden dimension: CTA c owns columns
//    [512 c, 512 c + 512) and keeps its 512 x 32 slice of Q resident in shared
//    memory as bf16 [Q_hi | Q_lo] (Q = Q_hi + Q_lo to about 2^-16).
//  * A token tile is 64 rows: the tensor-core products use M = 64, whose
//    accumulator rows occupy 16 of the 32 lanes of every TMEM lane quadrant.
//    The two tiles in flight take the two lane halves (lane offset 0 and 16)
//    of all 512 TMEM columns.
//  * A tile lands by TMA in one 64 KB landing buffer.  Three kinds of product
//    read it: the projection y = x [Q_hi | Q_lo] (N = 64, K = 512, into
//    columns 0-63 of the tile's lane half), and copies of x into the tile's
//    512 TMEM columns as fp32, by products with a 16 x 16 identity
//    (exact: every product is x * 1 and every sum has one nonzero term).
//    Slab 0's copy waits until y has been read out of columns 0-63.  Once
//    the copies are done the landing buffer takes the next tile, so the loads
//    run while the current tile's exchanges and passes go on.
//  * Projection exchange: each CTA's partial y of the 64 rows goes to shared
//    memory; after a cluster barrier the owner CTA of 64/CS rows pulls the CS
//    partials through distributed shared memory, sums them in a fixed order,
//    applies M and copies z (split bf16 hi/lo) into every CTA by bulk copy.
//  * The lift c = z_hi Q_hi^T + z_hi Q_lo^T + z_lo Q_hi^T (N = 2 x 256, K = 96)
//    accumulates onto the fp32 copy of x, so TMEM then holds the fp32 x_out.
//  * Pass 1 reads x_out from TMEM: row statistics (sum of squares folded
//    into float64, absmax) and bf16 x_out into a 64 KB staging buffer that TMA
//    stores back.  The statistics go to the row's owner (st.async), which
//    forms the scale and the row quantiser and pushes the quantiser to every
//    CTA.  Pass 2 reads x_out from TMEM again and writes the packed codes.
//  * One instruction stream for all 16 warps, software-pipelined over two
//    tiles: iteration k issues tile k's products, reads its partial
//    projection and starts its exchange, then runs pass 1 of tile k-1, the
//    owner statistics of tile k-1, the owner step of tile k's exchange and
//    pass 2 of tile k-1.  So each exchange's latency overlaps the other
//    tile's passes.
//  * Programmatic dependent launch: Q, M and the identity are staged before
//    the wait on the previous kernel of the stream; x and every output only
//    after it.
// Every mbarrier wait is bounded (2 s of %globaltimer).  A timeout sets a bit in
// the device status word, and the kernel keeps its barrier sequence so that no
// CTA is left waiting.  After a failed wait a thread issues no further
// asynchronous work, and the CTA drains what is in flight before freeing TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kTileM = 64;                    // token rows per tile (MMA M)
constexpr int kCols = 512;                    // hidden columns owned by one CTA
constexpr int kSlabCols = 64;                 // bf16 columns per 128-byte swizzle row
constexpr int kSlabs = kCols / kSlabCols;     // 8
constexpr int kSlabBytes = kTileM * 128;      // 8 KB
constexpr int kXBytes = kSlabs * kSlabBytes;  // 64 KB
constexpr int kQBytes = kCols * 128;          // 64 KB: 512 rows x [Q_hi(32) | Q_lo(32)] bf16
constexpr int kZBytes = kTileM * 128;         // 8 KB: partial y (fp32) / z hi|lo (bf16), per row
constexpr int kIdBytes = 16 * 128;            // 16 x 16 identity, in a 16-row SWIZZLE_128B block
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kTmemCols = 512;

struct PipeArgs {
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

// mbarriers.  "once per tile": completes once for every tile of the cluster;
// "[2]": one per tile parity, completes once every other tile.
enum : int {
    kBarLd = 0,               // [8] landing slab s (TMA), once per tile
    kBarY = kBarLd + kSlabs,  // projection done (commit), once per tile
    kBarId,                   // copies of slabs 1-7 done (commit), once per tile
    kBarS0,                   // copy of slab 0 done (commit), once per tile
    kBarZ,                    // [2] z of all rows in the operand buffer (owner warps + bulk copies)
    kBarC = kBarZ + 2,        // [2] lift done: TMEM holds x_out (commit)
    kBarSt = kBarC + 2,       // [2] owner: statistics of its rows from every CTA (st.async)
    kBarPrm = kBarSt + 2,     // [2] row quantisers of the tile (st.async)
    kNumBars = kBarPrm + 2
};

template <int CS>
struct PipeLayout {
    static constexpr int TPO = kTileM / CS;               // rows owned per CTA per tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffX = kOffQ + kQBytes;         // landing buffer
    static constexpr int kOffS = kOffX + kXBytes;         // x_out staging
    static constexpr int kOffI = kOffS + kXBytes;         // identity
    static constexpr int kOffZ = kOffI + kIdBytes;        // [2] operand buffers
    static constexpr int kOffM = kOffZ + 2 * kZBytes;     // M^T, 32 x 32 fp32, zero padded
    static constexpr int kOffSt = kOffM + 32 * 32 * 4;    // [2][CS source][TPO own rows] (ss, amax), 16 B
    static constexpr int kOffPrm = kOffSt + 2 * CS * TPO * 16;  // [2][64 rows] (inv, pre)
    static constexpr int kOffBar = kOffPrm + 2 * kTileM * 8;
    static constexpr int kOffTmem = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffTmem + 16;
    static constexpr int kSmem = kBytes + 1024;  // slack for 1024-byte alignment
    static_assert(kOffI % 1024 == 0 && kOffZ % 1024 == 0 && kZBytes % 1024 == 0, "swizzle atoms");
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

// Pass 1 on 32 consecutive fp32 x_out values: sum of squares (pairs), absmax
// (four partial maxima) and four 16-byte chunks of bf16 x_out into the staging
// row at chunks chunk0 .. chunk0 + 3.
__device__ __forceinline__ void pass1_block(const uint32_t (&v)[32], uint8_t *srow, int m, int chunk0, float2 &s2,
                                            float (&am)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 y = make_float2(__uint_as_float(v[c * 8 + 2 * e]), __uint_as_float(v[c * 8 + 2 * e + 1]));
            s2 = fma2(y, y, s2);
            am[e] = max3(am[e], fabsf(y.x), fabsf(y.y));
            o[e] = pack_bf16x2(y.x, y.y);
        }
        *reinterpret_cast<uint4 *>(srow + swz(m, chunk0 + c)) = make_uint4(o[0], o[1], o[2], o[3]);
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
k_align_pipe(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xo,
             const PipeArgs p) {
    using L = PipeLayout<CS>;
    constexpr int TPO = L::TPO;
    static_assert(CS * kCols <= 16384 && CS * TPO == kTileM && TPO <= kWarps, "cluster shape");
    constexpr bool kQuant = BITS > 0;  // BITS = 0: alignment only (x_out), no norm / codes
    constexpr uint32_t kZTx = uint32_t((CS - 1) * TPO * 128);  // z rows arriving from the other CTAs
    constexpr uint32_t kStTx = uint32_t(CS * TPO * 16);
    constexpr uint32_t kPrmTx = uint32_t(kTileM * 8);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = base + L::kOffQ;
    uint8_t *sx = base + L::kOffX;
    uint8_t *sstage = base + L::kOffS;
    uint8_t *sid = base + L::kOffI;
    uint8_t *szb = base + L::kOffZ;
    float *sm = reinterpret_cast<float *>(base + L::kOffM);
    uint8_t *sst = base + L::kOffSt;
    uint8_t *sprm = base + L::kOffPrm;
    const uint32_t bars = smem_u32(base + L::kOffBar);
    auto bar = [&](int i) { return bars + 8u * uint32_t(i); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + L::kOffTmem);
    auto zbuf = [&](int h) { return szb + h * kZBytes; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;  // TMEM lane quadrant; 128-column part
    const int hw = lane >> 4, rr = lane & 15;     // half-warp; row within the quadrant's 16
    const int m = 16 * quad + rr;                 // tile row of this thread
    const bool issuer = quad == 0 && lane == 0;   // x_out stores of its part's two slabs
    const uint32_t crank = cluster_ctarank();
    const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
    const int col0 = int(crank) * kCols;
    const int r = p.r;
    const int qmax = kQuant ? (1 << (BITS - 1)) - 1 : 1;
    const long long row_bytes = (long long)p.D * BITS / 8;
    const int R = p.rows_per_tile;
    int err = 0;

    asm volatile("griddepcontrol.launch_dependents;");
    auto tile_t0 = [&](int it) { return ((long long)cid + (long long)it * ncl) * R; };
    auto has_tile = [&](int it) { return it >= 0 && it < p.tiles_per_cluster && tile_t0(it) < p.T; };

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == kBarZ || i == kBarZ + 1) ? 1 + TPO : 1);
        fence_mbar_init();
        // the pushed exchanges of the first two tiles (each barrier is re-armed by
        // its waiter once the previous phase has completed)
        for (int h = 0; h < 2; ++h) {
            if (!has_tile(h)) continue;
            mbar_expect_tx(bar(kBarZ + h), kZTx);
            if (kQuant) {
                mbar_expect_tx(bar(kBarSt + h), kStTx);
                mbar_expect_tx(bar(kBarPrm + h), kPrmTx);
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

    // Q slice -> shared memory as [Q_hi | Q_lo] bf16 rows, SWIZZLE_128B; M -> 32x32
    // fp32 (transposed); the 16 x 16 identity; rows of the landing buffer that a
    // short tile never loads hold zeros.
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
    for (int idx = tid; idx < 32 * 32; idx += kThreads) {  // sm[k][j] = M[j][k]
        const int k = idx >> 5, j = idx & 31;
        sm[idx] = (j < r && k < r) ? __ldg(p.M + j * r + k) : 0.f;
    }
    for (int idx = tid; idx < kIdBytes / 16; idx += kThreads) {  // row n: 1.0 at column n < 16
        const int n = idx >> 3, ch = idx & 7;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (ch == (n >> 3)) w[(n & 7) >> 1] = (n & 1) ? 0x3F800000u : 0x00003F80u;
        *reinterpret_cast<uint4 *>(sid + n * 128 + swz(n, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int idx = tid; idx < kXBytes / 16; idx += kThreads)
        reinterpret_cast<uint4 *>(sx)[idx] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    cluster_sync();  // barriers initialised in every CTA before any push
    // Q, M and the identity are staged above while the previous kernel of the
    // stream may still run; x and every output only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const uint32_t slab_tx = uint32_t(R * 128);
    if (tid == 0 && has_tile(0)) {
#pragma unroll 1
        for (int s = 0; s < kSlabs; ++s) {
            mbar_expect_tx(bar(kBarLd + s), slab_tx);
            tma_load_2d(smem_u32(sx + s * kSlabBytes), &tm_x, col0 + s * kSlabCols, int(tile_t0(0)), bar(kBarLd + s));
        }
        if (has_tile(1)) {
            const int tn = int(tile_t0(1));
#pragma unroll 1
            for (int s = 0; s < kSlabs; ++s) tma_prefetch_2d(&tm_x, col0 + s * kSlabCols, tn);
        }
    }

    const uint32_t idesc_y = idesc_bf16_f32(64, 64, false, true);
    const uint32_t idesc_i = idesc_bf16_f32(64, 16, false, false);
    const uint32_t idesc_c = idesc_bf16_f32(64, 256, false, false);
    // (A K-step, B K-step) pairs of the lift: z_hi Q_hi^T, z_hi Q_lo^T, z_lo Q_hi^T
    constexpr uint32_t kA[6] = {0, 1, 0, 1, 2, 3}, kB[6] = {0, 1, 2, 3, 0, 1};

#pragma unroll 1
    for (int it = 0; it <= p.tiles_per_cluster; ++it) {
        const int h = it & 1, hp = h ^ 1;            // TMEM lane half / buffers of tiles it and it-1
        const bool cur = has_tile(it), prev = has_tile(it - 1);
        const uint32_t ph1 = uint32_t(it) & 1u;      // phase of the once-per-tile barriers
        const uint32_t php = uint32_t((it - 1) >> 1) & 1u;  // phase of parity-hp barriers, tile it-1
        const uint32_t dh = tmem + (uint32_t(16 * h) << 16);    // D address of tile it
        const uint32_t dp = tmem + (uint32_t(16 * hp) << 16);   // D address of tile it-1
        const long long t0p = tile_t0(it - 1);

        // ---- A (thread 0): projection and copies of tile it, lift of tile it-1
        if (tid == 0) {
            const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(sx), 1024));
            const uint64_t bq0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
            if (cur) {
#pragma unroll 1
                for (int s = 0; s < kSlabs; ++s) {
                    if (!mbar_wait(bar(kBarLd + s), ph1, err != 0)) err |= kErrMbarTimeout;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // K steps of 16 columns, 32 bytes apart
                        const int i = 4 * s + k;
                        if (!err) umma_f16(dh, ad0 + (uint32_t(s * kSlabBytes + k * 32) >> 4),
                                           bq0 + (uint32_t(i * 2048) >> 4), idesc_y, i != 0);
                    }
                }
                if (!err) umma_commit(bar(kBarY));
                const uint64_t bi = opaque(smem_desc_sw128(smem_u32(sid), 1024));
#pragma unroll 1
                for (int s = 1; s < kSlabs; ++s) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (!err) umma_f16(dh + uint32_t(64 * s + 16 * j),
                                           ad0 + (uint32_t(s * kSlabBytes + j * 32) >> 4), bi, idesc_i, 0);
                }
                if (!err) umma_commit(bar(kBarId));
            }
            if (prev) {
                if (!mbar_wait(bar(kBarZ + hp), php, err != 0)) err |= kErrMbarTimeout;
                if (has_tile(it + 1)) mbar_expect_tx(bar(kBarZ + hp), kZTx);
                tc_fence_after();
                fence_proxy_async();
                const uint64_t az = opaque(smem_desc_sw128(smem_u32(zbuf(hp)), 1024));
#pragma unroll
                for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
                    for (int s = 0; s < 6; ++s)
                        if (!err) umma_f16(dp + uint32_t(nh * 256), az + ((kA[s] * 32) >> 4),
                                           bq0 + ((uint32_t(nh) * 32768 + kB[s] * 32) >> 4), idesc_c, 1);
                }
                if (!err) umma_commit(bar(kBarC + hp));
            }
        }
        __syncwarp();

        // ---- B: partial projection of tile it (part-0 warps) -> operand buffer;
        // copy of slab 0; the next tile's loads
        if (cur && part == 0) {
            if (!mbar_wait(bar(kBarY), ph1, err != 0)) err |= kErrMbarTimeout;
            tc_fence_after();
            uint32_t a[32];
            tmem_ld16x2<32>(dh + (uint32_t(32 * quad) << 16), a);  // half 0: y_hi part, half 1: y_lo part
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float own = __uint_as_float(a[k]);
                a[k] = __float_as_uint(own + __shfl_xor_sync(0xFFFFFFFFu, own, 16));
            }
            uint8_t *prow = zbuf(h) + m * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // half-warp hw writes 16-byte chunks 4 hw .. 4 hw + 3
                const uint4 lo4 = make_uint4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
                const uint4 hi4 = make_uint4(a[16 + 4 * c], a[17 + 4 * c], a[18 + 4 * c], a[19 + 4 * c]);
                *reinterpret_cast<uint4 *>(prow + swz(m, 4 * hw + c)) = hw ? hi4 : lo4;
            }
            tc_fence_before();
            named_sync(2, 128);  // the four part-0 warps: y read out of columns 0-63
            if (tid == 0) {
                tc_fence_after();
                const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(sx), 1024));
                const uint64_t bi = opaque(smem_desc_sw128(smem_u32(sid), 1024));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (!err) umma_f16(dh + uint32_t(16 * j), ad0 + (uint32_t(j * 32) >> 4), bi, idesc_i, 0);
                if (!err) umma_commit(bar(kBarS0));
                if (has_tile(it + 1)) {
                    const int tn = int(tile_t0(it + 1));
                    if (!mbar_wait(bar(kBarId), ph1, err != 0)) err |= kErrMbarTimeout;
#pragma unroll 1
                    for (int s = 1; s < kSlabs; ++s) {
                        mbar_expect_tx(bar(kBarLd + s), slab_tx);
                        if (!err) tma_load_2d(smem_u32(sx + s * kSlabBytes), &tm_x, col0 + s * kSlabCols, tn,
                                              bar(kBarLd + s));
                    }
                    if (!mbar_wait(bar(kBarS0), ph1, err != 0)) err |= kErrMbarTimeout;
                    mbar_expect_tx(bar(kBarLd), slab_tx);
                    if (!err) tma_load_2d(smem_u32(sx), &tm_x, col0, tn, bar(kBarLd));
                    if (has_tile(it + 2)) {
                        const int tn2 = int(tile_t0(it + 2));
#pragma unroll 1
                        for (int s = 0; s < kSlabs; ++s) tma_prefetch_2d(&tm_x, col0 + s * kSlabCols, tn2);
                    }
                }
            }
            __syncwarp();
        }
        tc_fence_before();
        cluster_arrive();  // partial projections of tile it visible cluster-wide

        // ---- C: pass 1 of tile it-1: x_out from TMEM -> statistics; bf16 x_out ->
        // staging -> TMA store (two slabs per column part)
        if (prev) {
            if (issuer) bulk_wait_read0();  // this part's previous stores have read the staging
            named_sync(3 + part, 128);
            if (!mbar_wait(bar(kBarC + hp), php, err != 0)) err |= kErrMbarTimeout;
            tc_fence_after();
            const uint32_t taddr = dp + (uint32_t(32 * quad) << 16) + uint32_t(128 * part);
            uint32_t va[32], vb[32];
            tmem_ld16x2<64>(taddr, va);       // columns 128 part + 64 hw + (0..31)
            tmem_ld16x2<64>(taddr + 32, vb);  // columns 128 part + 64 hw + (32..63)
            tmem_wait_ld();
            float2 s2 = make_float2(0.f, 0.f);
            float am[4] = {0.f, 0.f, 0.f, 0.f};
            uint8_t *srow = sstage + (2 * part + hw) * kSlabBytes + m * 128;
            pass1_block(va, srow, m, 0, s2, am);
            double ss = double(s2.x) + double(s2.y);
            s2 = make_float2(0.f, 0.f);
            pass1_block(vb, srow, m, 4, s2, am);
            ss += double(s2.x) + double(s2.y);
            float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
            fence_proxy_async_cta();  // staging (generic writes) -> TMA store (async proxy)
            named_sync(3 + part, 128);
            if (issuer) {
                if (!err) {
                    tma_store_2d(&tm_xo, smem_u32(sstage + 2 * part * kSlabBytes), col0 + 128 * part, int(t0p));
                    tma_store_2d(&tm_xo, smem_u32(sstage + (2 * part + 1) * kSlabBytes), col0 + 128 * part + 64,
                                 int(t0p));
                }
                bulk_commit();
            }
            if (kQuant) {
                ss += __shfl_xor_sync(0xFFFFFFFFu, ss, 16);
                amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 16));
                // parts 1-3 leave the row's partial in the tile's operand buffer (free:
                // its lift has completed); part 0 folds them
                uint8_t *scr = zbuf(hp);
                if (part > 0 && hw == 0) {
                    reinterpret_cast<double *>(scr + ((part - 1) * kTileM + m) * 16)[0] = ss;
                    reinterpret_cast<float *>(scr + ((part - 1) * kTileM + m) * 16)[2] = amax;
                }
                named_sync(1, kThreads);
                if (part == 0 && hw == 0) {
#pragma unroll
                    for (int k = 0; k < 3; ++k) {
                        ss += reinterpret_cast<const double *>(scr + (k * kTileM + m) * 16)[0];
                        amax = fmaxf(amax, reinterpret_cast<const float *>(scr + (k * kTileM + m) * 16)[2]);
                    }
                    const uint32_t owner = uint32_t(m / TPO);
                    const uint32_t dst = smem_u32(sst + ((hp * CS + int(crank)) * TPO + m % TPO) * 16);
                    if (!err) st_async_v4(mapa(dst, owner), uint32_t(__double2loint(ss)), uint32_t(__double2hiint(ss)),
                                          __float_as_uint(amax), 0u, mapa(bar(kBarSt + hp), owner));
                }
            }
        }

        // ---- D: owner: totals of its rows of tile it-1 over the cluster in a fixed
        // order (deterministic), scale, row quantiser pushed to every CTA
        if (kQuant && prev && tid < CS * TPO) {
            const int rl = tid / CS, dst_cta = tid % CS;
            if (!mbar_wait(bar(kBarSt + hp), php, err != 0)) err |= kErrMbarTimeout;
            double ss_t = 0.0;
            float am_t = 0.f;
#pragma unroll
            for (int c = 0; c < CS; ++c) {
                const float4 v = *reinterpret_cast<const float4 *>(sst + ((hp * CS + c) * TPO + rl) * 16);
                ss_t += __hiloint2double(__float_as_int(v.y), __float_as_int(v.x));
                am_t = fmaxf(am_t, v.z);
            }
            const int mo = int(crank) * TPO + rl;
            const float ms = float(ss_t / double(p.D));
            const float rs = 1.0f / sqrtf(ms + p.eps);
            const RowQuant q = row_quant(am_t, qmax);
            if (dst_cta == 0 && mo < R && t0p + mo < p.T) p.scales[t0p + mo] = am_t > 0.f ? (am_t * rs) / float(qmax) : 0.f;
            if (!err) st_async_v2(mapa(smem_u32(sprm + (hp * kTileM + mo) * 8), uint32_t(dst_cta)),
                                  __float_as_uint(q.inv), __float_as_uint(q.pre), mapa(bar(kBarPrm + hp), uint32_t(dst_cta)));
            if (tid == 0 && has_tile(it + 1)) mbar_expect_tx(bar(kBarSt + hp), kStTx);
        }

        cluster_wait();

        // ---- E: owner CTA of tile it's rows: sum the partials (one warp per row,
        // one projection entry per lane), z = M y, z hi|lo pushed to every CTA
        if (cur && warp < TPO) {
            const int kq = lane;
            const int mo = int(crank) * TPO + warp;
            const uint32_t row_addr = smem_u32(zbuf(h) + mo * 128);
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
            uint32_t hwd[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) hwd[e] = (__shfl_sync(0xFFFFFFFFu, hl, src0 + e) >> sh) & 0xFFFFu;
            const uint32_t w0 = hwd[0] | (hwd[1] << 16), w1 = hwd[2] | (hwd[3] << 16);
            const uint32_t w2 = hwd[4] | (hwd[5] << 16), w3 = hwd[6] | (hwd[7] << 16);
            // the row goes into this CTA's operand buffer (its own partial has been
            // read above), then by bulk copy into the same row of every other CTA
            if (lane < 8) *reinterpret_cast<uint4 *>(zbuf(h) + mo * 128 + swz(mo, ch)) = make_uint4(w0, w1, w2, w3);
            fence_proxy_async_cta();
            __syncwarp();
            if (lane < CS && lane != int(crank))
                if (!err) bulk_copy_to_cluster(mapa(row_addr, uint32_t(lane)), row_addr, 128u,
                                               mapa(bar(kBarZ + h), uint32_t(lane)));
            if (lane == 0) mbar_arrive(bar(kBarZ + h));
        }

        // ---- F: pass 2 of tile it-1: codes from the fp32 x_out in TMEM
        if constexpr (kQuant) {
        if (prev) {
            if (!mbar_wait(bar(kBarPrm + hp), php, err != 0)) err |= kErrMbarTimeout;
            const RowQuant rq{reinterpret_cast<const float *>(sprm + (hp * kTileM + m) * 8)[0],
                              reinterpret_cast<const float *>(sprm + (hp * kTileM + m) * 8)[1]};
            tc_fence_after();
            const uint32_t taddr = dp + (uint32_t(32 * quad) << 16) + uint32_t(128 * part);
            uint32_t va[32], vb[32];
            tmem_ld16x2<64>(taddr, va);
            tmem_ld16x2<64>(taddr + 32, vb);
            tmem_wait_ld();
            uint32_t words[2 * BITS];
            code_block<BITS>(va, rq, words);
            code_block<BITS>(vb, rq, words + BITS);
            if (m < R && t0p + m < p.T) {
                uint8_t *dst = p.codes + (t0p + m) * row_bytes + (long long)(col0 + 128 * part + 64 * hw) * BITS / 8;
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
            if (tid == 0 && has_tile(it + 1)) mbar_expect_tx(bar(kBarPrm + hp), kPrmTx);
        }
        }

        // ---- G: TMEM lane half of tile it-1 read for the last time; the next
        // iteration's products may overwrite it
        tc_fence_before();
        named_sync(1, kThreads);
        tc_fence_after();
    }
    if (issuer) bulk_wait0();

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
        void *q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(q);
    }
    return fn;
}

bool make_map(CUtensorMap *mp, const void *ptr, long long T, int D, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kSlabCols), cuuint32_t(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int CS, int BITS>
struct PipeKernel {
    static int max_clusters[64];
    static bool configured[64];

    static cudaError_t configure(int dev) {
        if (configured[dev]) return cudaSuccess;
        auto kern = k_align_pipe<CS, BITS>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PipeLayout<CS>::kSmem);
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
        cfg.dynamicSmemBytes = PipeLayout<CS>::kSmem;
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
        PipeArgs a;
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
        cfg.dynamicSmemBytes = PipeLayout<CS>::kSmem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_align_pipe<CS, BITS>, mx, mxo, a);
        if (e == cudaSuccess) {
            *launched = true;
            count_launch();
        }
        return e;
    }
};

template <int CS, int BITS>
int PipeKernel<CS, BITS>::max_clusters[64];
template <int CS, int BITS>
bool PipeKernel<CS, BITS>::configured[64];

}  // namespace

bool align_pipe_supports(int D, int r, int dtype, long long T) {
    return dtype == 1 && (D == 4096 || D == 8192) && r >= 1 && r <= 32 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_align_pipe(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                              float *scales, long long T, int D, int r, int bits, float eps, cudaStream_t s,
                              bool *launched) {
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    if (D == 4096) {
        if (bits == 0) return PipeKernel<8, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
        return bits == 4 ? PipeKernel<8, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched)
                         : PipeKernel<8, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    }
    if (bits == 0) return PipeKernel<16, 0>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
    return bits == 4 ? PipeKernel<16, 4>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched)
                     : PipeKernel<16, 3>::launch(x, Q, M, x_out, codes, scales, T, D, r, eps, status, s, launched);
}

}  // namespace rsq
