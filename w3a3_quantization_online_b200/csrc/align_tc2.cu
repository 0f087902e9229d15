// align_tc2.cu -- double-buffered tensor-core residual subspace alignment fused
// with the weight-free RMSNorm and the per-token symmetric quantiser, for a
// hidden size of 4096, bf16 I/O.
//
// ReSpinQuant paper notes, key design 3: y = Q^T x (D -> r), z = M y,
// x_out = x + Q z.  Infra Quant II, QuaRot / Method: scale-free RMSNorm in FP32
// and per-token symmetric absmax quantisation (SpinQuant / Motivation:
// alpha = max|X| / (2^(N-1) - 1)).
//
// Same arithmetic as align_tc.cu (bf16 hi/lo split of Q and z, fp32 TMEM
// accumulators, DSMEM reductions), but organised so that two token tiles are in
// flight in every CTA:
//  * a cluster of 16 CTAs splits the 4096 columns; each CTA owns 256 columns,
//    so one 128-row tile needs 64 KB of shared memory and 256 TMEM columns, and
//    two tiles fit (two TMA buffers, two TMEM regions);
//  * iteration i finishes tile i (pass 1: x_out and statistics; pass 2: codes)
//    while tile i+1 goes through its projection, cluster reduction and lift:
//      - tile i+1's first product (y) runs on the tensor core during pass 1(i);
//      - one cluster barrier publishes both the statistics of tile i and the
//        partial projections of tile i+1, then the totals of tile i and the z
//        of tile i+1 are computed from them;
//      - a second barrier publishes z(i+1); it is split into arrive / wait with
//        pass 2(i) in between, and tile i+1's second product (c) is issued
//        right after it;
//  * the x_out store of tile i (TMA) is issued between the arrive and the wait
//    of the first barrier, so the barrier's release never waits for it, and the
//    next tile's load goes into the buffer as soon as that store has read it.
// Every mbarrier wait is bounded and reported through the device status word.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int CS = 16;                       // CTAs per cluster
constexpr int kTileM = 128;                  // token rows per tile
constexpr int kCols = 256;                   // hidden columns per CTA
constexpr int kSlabCols = 64;
constexpr int kSlabs = kCols / kSlabCols;    // 4
constexpr int kSlabBytes = kTileM * 128;     // 16 KB
constexpr int kXBytes = kSlabs * kSlabBytes; // 64 KB per tile buffer
constexpr int kQBytes = kCols * 128;         // 32 KB: [Q_hi | Q_lo] bf16 rows
constexpr int kZBytes = kTileM * 128;        // 16 KB: partial y (fp32) / z hi|lo (bf16)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kHalfCols = kCols / 2;         // columns per thread
constexpr int kTPO = kTileM / CS;            // rows reduced by each CTA (8): one warp per row
constexpr int kOffX = 0;
constexpr int kOffQ = kOffX + 2 * kXBytes;
constexpr int kOffZ = kOffQ + kQBytes;
constexpr int kOffM = kOffZ + kZBytes;        // M^T, 32 x 32 fp32
constexpr int kOffYred = kOffM + 32 * 32 * 4; // kTPO x 32 fp32
constexpr int kOffStat = kOffYred + kTPO * 32 * 4;
constexpr int kOffLoc = kOffStat + kTileM * 16;
constexpr int kOffBar = kOffLoc + kTileM * 16;
constexpr int kNumBars = 4;                   // load[2], y, c
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffTmem + 16 + 1024;

struct Args {
    const float *Q;
    const float *M;
    uint8_t *codes;
    float *scales;
    int *status;
    long long T;
    int r;
    int tiles_per_cluster;
    int codes_v8;  // codes pointer is 32-byte aligned: 256-bit stores
    float eps;
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

// x_out = x + c for one 32-column block (see align_tc.cu).
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

template <int BITS>
__device__ __forceinline__ void code_block(const uint32_t (&v)[32], const RowQuant &rq, bool scaled,
                                           uint32_t *words) {
    uint32_t g[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[gi * 8 + e]);
        g[gi] = pack8_fast<BITS>(f, rq.inv, rq.pre, scaled);
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

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
k_align_tc_db(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xo, const Args p) {
    constexpr int D = CS * kCols;
    constexpr int qmax = (1 << (BITS - 1)) - 1;
    constexpr long long row_bytes = (long long)D * BITS / 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = base + kOffQ;
    uint8_t *sz = base + kOffZ;
    float *sm = reinterpret_cast<float *>(base + kOffM);
    float *syred = reinterpret_cast<float *>(base + kOffYred);
    uint8_t *sstat = base + kOffStat;
    uint8_t *sloc = base + kOffLoc;
    const uint32_t bar_load0 = smem_u32(base + kOffBar);  // + 8 * buffer
    const uint32_t bar_y = bar_load0 + 16, bar_c = bar_load0 + 24;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffTmem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const uint32_t cid = cluster_id_x(), ncl = ncluster_x();
    const int col0 = int(crank) * kCols;
    const int r = p.r;
    const int R = kTileM;
    int err = 0;

    if (tid == 0) {
        mbar_init(bar_load0, 1);
        mbar_init(bar_load0 + 8, 1);
        mbar_init(bar_y, 1);
        mbar_init(bar_c, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    if (tid == 32) {
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_xo);
    }
    // Q slice -> [Q_hi | Q_lo] bf16 rows (SWIZZLE_128B); M^T -> fp32 32 x 32
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
    for (int idx = tid; idx < 32 * 32; idx += kThreads) {
        const int k = idx >> 5, j = idx & 31;
        sm[idx] = (j < r && k < r) ? __ldg(p.M + j * r + k) : 0.f;
    }
    fence_proxy_async_cta();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    cluster_sync();

    // tiles of this cluster: cid, cid + ncl, ... (all CTAs of a cluster agree)
    int n = 0;
    for (int it = 0; it < p.tiles_per_cluster; ++it)
        if (((long long)cid + (long long)it * ncl) * R < p.T) n = it + 1;
    auto tile_t0 = [&](int i) { return ((long long)cid + (long long)i * ncl) * R; };
    auto xbuf = [&](int i) { return base + kOffX + (i & 1) * kXBytes; };
    auto issue_load = [&](int i) {  // thread 0
        const uint32_t bar = bar_load0 + 8 * (i & 1);
        mbar_expect_tx(bar, uint32_t(kXBytes));
#pragma unroll
        for (int s = 0; s < kSlabs; ++s)
            if (!err) tma_load_2d(smem_u32(xbuf(i) + s * kSlabBytes), &tm_x, col0 + s * kSlabCols, int(tile_t0(i)), bar);
    };

    const int quad = warp & 3, half = warp >> 2;
    const int m = quad * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t idesc_y = idesc_bf16_f32(128, 64, false, true);
    const uint32_t idesc_c = idesc_bf16_f32(128, 256, false, false);
    auto region = [&](int i) { return uint32_t((i & 1) * 256); };

    auto mma1 = [&](int i) {  // thread 0: y(i) = x(i) [Q_hi | Q_lo] into region(i) columns [0, 64)
        tc_fence_after();
        const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(xbuf(i)), 1024));
        const uint64_t bd0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
#pragma unroll
        for (int k = 0; k < kSlabs * 4; ++k)
            if (!err) umma_f16(tmem + region(i), ad0 + (uint32_t((k >> 2) * kSlabBytes + (k & 3) * 32) >> 4),
                     bd0 + (uint32_t(k * 2048) >> 4), idesc_y, k != 0);
        if (!err) umma_commit(bar_y);
    };
    auto mma2 = [&](int i) {  // thread 0: c(i) = z_hi Q_hi^T + z_hi Q_lo^T + z_lo Q_hi^T into region(i)
        tc_fence_after();
        fence_proxy_async();
        const uint64_t ad0 = opaque(smem_desc_sw128(smem_u32(sz), 1024));
        const uint64_t bd0 = opaque(smem_desc_sw128(smem_u32(sq), 1024));
        constexpr uint32_t kA[6] = {0, 1, 0, 1, 2, 3}, kB[6] = {0, 1, 2, 3, 0, 1};
#pragma unroll
        for (int s = 0; s < 6; ++s)
            if (!err) umma_f16(tmem + region(i), ad0 + ((kA[s] * 32) >> 4), bd0 + ((kB[s] * 32) >> 4), idesc_c, s != 0);
        if (!err) umma_commit(bar_c);
    };
    auto yread = [&](int i) {  // warps 0-3: partial y of row m -> P rows (swizzled fp32)
        if (half == 0) {
            uint32_t a[32], b[32];
            tmem_ld32(tmem + lane_base + region(i), a);
            tmem_ld32(tmem + lane_base + region(i) + 32, b);
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
    };
    auto owner = [&]() {  // this CTA's kTPO rows: sum the CS partials, z = M y, scatter z hi|lo
        const int mloc = warp, kq = lane;  // one warp per row, one projection entry per lane
        const int mo = int(crank) * kTPO + mloc;
        const uint32_t row_addr = smem_u32(sz + mo * 128);
        float pv[CS];
#pragma unroll
        for (int c = 0; c < CS; ++c) pv[c] = ld_dsmem_f32(mapa(row_addr, uint32_t(c)) + swz(mo, kq >> 2) + 4 * (kq & 3));
        float y = 0.f;
#pragma unroll
        for (int c = 0; c < CS; ++c) y += pv[c];
        syred[mloc * 32 + kq] = y;
        __syncwarp();
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) acc = fmaf(sm[k * 32 + kq], syred[mloc * 32 + k], acc);
        const uint16_t hi = bf16_bits(acc), lo = bf16_bits(acc - bf16_val(bf16_bits(acc)));
        __syncwarp();
#pragma unroll
        for (int c = 0; c < CS; ++c) {
            const uint32_t ra = mapa(row_addr, uint32_t(c));
            st_dsmem_u16(ra + swz(mo, kq >> 3) + 2 * (kq & 7), hi);
            st_dsmem_u16(ra + swz(mo, 4 + (kq >> 3)) + 2 * (kq & 7), lo);
        }
    };

    // ---------------------------------------------------------------- prologue: tile 0 to its lift
    if (n > 0) {
        if (tid == 0) {
            issue_load(0);
            if (n > 1) issue_load(1);
        }
        if (!mbar_wait(bar_load0, 0, err != 0)) err |= kErrMbarTimeout;
        if (tid == 0) mma1(0);
        if (!mbar_wait(bar_y, 0, err != 0)) err |= kErrMbarTimeout;
        tc_fence_after();
        yread(0);
        tc_fence_before();
        cluster_sync();
        owner();
        fence_proxy_async();
        cluster_sync();
        if (tid == 0) mma2(0);
    }

    float pend_scale = 0.f;
    float *pend_scale_at = nullptr;
    for (int i = 0; i < n; ++i) {
        const bool nx = i + 1 < n;
        const long long t0 = tile_t0(i);
        const int nrows = int(p.T - t0 < R ? p.T - t0 : R);

        // A: next tile's projection runs on the tensor core during pass 1
        if (nx) {
            if (!mbar_wait(bar_load0 + 8 * ((i + 1) & 1), uint32_t(((i + 1) >> 1) & 1), err != 0)) err |= kErrMbarTimeout;
            if (tid == 0) mma1(i + 1);
        }
        // B/C: pass 1 of tile i
        if (!mbar_wait(bar_c, uint32_t(i & 1), err != 0)) err |= kErrMbarTimeout;
        tc_fence_after();
        double ss = 0.0;
        float amax = 0.f;
        {
            float2 s2 = make_float2(0.f, 0.f);
            float am[4] = {0.f, 0.f, 0.f, 0.f};
            constexpr int kBlocks = kHalfCols / 32;  // 4
            uint32_t va[32], vb[32];
            const uint32_t taddr = tmem + lane_base + region(i) + uint32_t(half * kHalfCols);
            uint8_t *xb = xbuf(i) + m * 128;
            tmem_ld32(taddr, va);
            tmem_wait_ld();
#pragma unroll
            for (int b = 0; b < kBlocks; b += 2) {
                const int cb = half * kBlocks + b;  // 32-column block within the CTA slice
                tmem_wait_st();
                tmem_ld32(taddr + (b + 1) * 32, vb);
                xout_block(va, xb + (cb >> 1) * kSlabBytes, m, (cb & 1) * 4, s2, am);
                tmem_st32(taddr + b * 32, va);
                tmem_wait_ld();
                tmem_wait_st();
                if (b + 2 < kBlocks) tmem_ld32(taddr + (b + 2) * 32, va);
                xout_block(vb, xb + ((cb + 1) >> 1) * kSlabBytes, m, ((cb + 1) & 1) * 4, s2, am);
                tmem_st32(taddr + (b + 1) * 32, vb);
                tmem_wait_ld();
                ss += double(s2.x) + double(s2.y);
                s2 = make_float2(0.f, 0.f);
            }
            tmem_wait_st();
            amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
        }
        fence_proxy_async_cta();  // x_out (generic writes) -> TMA store
        // D: fold the two column halves of each row into one entry
        if (half == 1) {
            reinterpret_cast<double *>(sloc + m * 16)[0] = ss;
            reinterpret_cast<float *>(sloc + m * 16)[2] = amax;
        }
        named_sync(1, kThreads);
        if (half == 0) {
            ss += reinterpret_cast<const double *>(sloc + m * 16)[0];
            amax = fmaxf(amax, reinterpret_cast<const float *>(sloc + m * 16)[2]);
            reinterpret_cast<double *>(sstat + m * 16)[0] = ss;
            reinterpret_cast<float *>(sstat + m * 16)[2] = amax;
        }
        // E: partial projection of the next tile (its product finished during pass 1)
        if (nx) {
            if (!mbar_wait(bar_y, uint32_t((i + 1) & 1), err != 0)) err |= kErrMbarTimeout;
            tc_fence_after();
            yread(i + 1);
        }
        tc_fence_before();
        // F/G: publish statistics(i) and partials(i+1); store x_out(i) while the barrier settles
        cluster_arrive();
        if (tid == 0) {
#pragma unroll
            for (int s = 0; s < kSlabs; ++s)
                if (!err) tma_store_2d(&tm_xo, smem_u32(xbuf(i) + s * kSlabBytes), col0 + s * kSlabCols, int(t0));
            bulk_commit();
        }
        cluster_wait();
        // H: row totals of tile i (half 0), z of tile i+1 (owner rows)
        if (half == 0) {
            float4 sv[CS];
#pragma unroll
            for (int c = 0; c < CS; ++c) sv[c] = ld_dsmem_f4(mapa(smem_u32(sstat + m * 16), uint32_t(c)));
            double ss_t = 0.0;
            float am_t = 0.f;
#pragma unroll
            for (int c = 0; c < CS; ++c) {
                ss_t += __hiloint2double(__float_as_int(sv[c].y), __float_as_int(sv[c].x));
                am_t = fmaxf(am_t, sv[c].z);
            }
            const float ms = float(ss_t / double(D));
            const float rs = 1.0f / sqrtf(ms + p.eps);
            const RowQuant q = row_quant(am_t, qmax);
            if (crank == 0 && m < nrows) {
                pend_scale = am_t > 0.f ? (am_t * rs) / float(qmax) : 0.f;
                pend_scale_at = p.scales + t0 + m;
            }
            reinterpret_cast<float *>(sloc + m * 16)[0] = q.inv;
            reinterpret_cast<float *>(sloc + m * 16)[1] = q.pre;
        }
        if (nx) owner();
        fence_proxy_async();
        // I: publish z(i+1); pass 2(i) runs while the barrier settles
        cluster_arrive();
        named_sync(1, kThreads);
        if (tid == 0) {  // the tile buffer is free once TMA has read x_out(i)
            bulk_wait_read0();
            if (i + 2 < n) issue_load(i + 2);
        }
        {
            RowQuant rq;
            rq.inv = reinterpret_cast<const float *>(sloc + m * 16)[0];
            rq.pre = reinterpret_cast<const float *>(sloc + m * 16)[1];
            const bool scaled = rq.pre != 1.0f;
            constexpr int kBlocks = kHalfCols / 32;  // 4
            uint32_t words[BITS * kBlocks];          // 128 codes: 64 B (INT4) / 48 B (INT3)
            const uint32_t taddr = tmem + lane_base + region(i) + uint32_t(half * kHalfCols);
            uint32_t va[32], vb[32];
            tmem_ld32(taddr, va);
            tmem_wait_ld();
#pragma unroll
            for (int b = 0; b < kBlocks; b += 2) {
                tmem_ld32(taddr + (b + 1) * 32, vb);
                code_block<BITS>(va, rq, scaled, words + b * BITS);
                tmem_wait_ld();
                if (b + 2 < kBlocks) tmem_ld32(taddr + (b + 2) * 32, va);
                code_block<BITS>(vb, rq, scaled, words + (b + 1) * BITS);
                tmem_wait_ld();
            }
            if (m < nrows) {
                uint8_t *dst = p.codes + (t0 + m) * row_bytes + (long long)(col0 + half * kHalfCols) * BITS / 8;
                if (BITS == 4 && p.codes_v8) {  // 64 B at a 32-byte boundary
                    st_global_v8(dst, words);
                    st_global_v8(dst + 32, words + 8);
                } else if (BITS == 4) {
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        reinterpret_cast<uint4 *>(dst)[w] =
                            make_uint4(words[4 * w], words[4 * w + 1], words[4 * w + 2], words[4 * w + 3]);
                } else {  // 48 B, 16-byte aligned
#pragma unroll
                    for (int w = 0; w < 3; ++w)
                        reinterpret_cast<uint4 *>(dst)[w] =
                            make_uint4(words[4 * w], words[4 * w + 1], words[4 * w + 2], words[4 * w + 3]);
                }
            }
        }
        cluster_wait();
        if (pend_scale_at) {  // after the barrier, so that its release does not wait for it
            *pend_scale_at = pend_scale;
            pend_scale_at = nullptr;
        }
        // M: the next tile's lift
        if (nx && tid == 0) mma2(i + 1);
        tc_fence_before();
        named_sync(1, kThreads);  // TMEM region(i) and sloc reads done
    }

    if (tid == 0) bulk_wait0();
    tc_fence_before();
    // after a failed wait no further asynchronous work was issued: let what was
    // already in flight land before TMEM is freed and the CTA exits
    if (__syncthreads_or(err)) drain_delay();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
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
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

bool make_map(CUtensorMap *map, const void *ptr, long long T, int D) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kSlabCols), cuuint32_t(kTileM)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS>
struct DbKernel {
    static int max_clusters[64];
    static bool configured[64];

    static cudaError_t configure(int dev) {
        if (configured[dev]) return cudaSuccess;
        auto kern = k_align_tc_db<BITS>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(CS, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nc = 0;
        e = cudaOccupancyMaxActiveClusters(&nc, kern, &cfg);
        if (e != cudaSuccess) return e;
        max_clusters[dev] = nc;
        configured[dev] = true;
        return cudaSuccess;
    }

    static cudaError_t launch(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                              float *scales, long long T, int r, float eps, int *status, cudaStream_t s,
                              bool *launched) {
        *launched = false;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaSuccess;
        e = configure(dev);
        if (e != cudaSuccess) return e;
        const int maxcl = max_clusters[dev];
        if (maxcl < 1) return cudaSuccess;
        const long long tiles = (T + kTileM - 1) / kTileM;
        const int ncl = int(tiles < maxcl ? tiles : maxcl);
        const int tpc = int((tiles + ncl - 1) / ncl);
        CUtensorMap mx, mxo;
        if (!make_map(&mx, x, T, CS * kCols) || !make_map(&mxo, x_out, T, CS * kCols)) return cudaErrorInvalidValue;
        Args a;
        a.Q = Q;
        a.M = M;
        a.codes = codes;
        a.scales = scales;
        a.status = status;
        a.T = T;
        a.r = r;
        a.tiles_per_cluster = tpc;
        a.codes_v8 = (reinterpret_cast<uintptr_t>(codes) & 31u) == 0;
        a.eps = eps;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(CS * ncl, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_align_tc_db<BITS>, mx, mxo, a);
        if (e == cudaSuccess) {
            *launched = true;
            count_launch();
        }
        return e;
    }
};

template <int BITS>
int DbKernel<BITS>::max_clusters[64];
template <int BITS>
bool DbKernel<BITS>::configured[64];

}  // namespace

bool align_tc_db_supports(int D, int r, int dtype, long long T) {
    return dtype == 1 && D == CS * kCols && r >= 1 && r <= 32 && T >= 1 && T <= 0x7FFFFFFFLL;
}

cudaError_t launch_align_tc_db(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                               float *scales, long long T, int r, int bits, float eps, cudaStream_t s,
                               bool *launched) {
    int *status = device_status_word();
    if (!status) return cudaErrorInvalidDevice;
    return bits == 4 ? DbKernel<4>::launch(x, Q, M, x_out, codes, scales, T, r, eps, status, s, launched)
                     : DbKernel<3>::launch(x, Q, M, x_out, codes, scales, T, r, eps, status, s, launched);
}

}  // namespace rsq
