// align_decode.cu -- residual subspace alignment + RMSNorm + quantiser for a
// handful of token rows (decode: T <= 32), where a per-tile pipeline cannot be
// filled and the latency of the chain of reductions is all that counts.
//
// ReSpinQuant paper notes, key design 3: y = Q^T x, z = M y, x_out = x + Q z.
// Infra Quant II, QuaRot / Method: scale-free RMSNorm in FP32, per-token
// symmetric absmax quantisation.
//
// One cluster of 16 CTAs splits the hidden dimension (CTA c owns columns
// [c D/16, (c+1) D/16)) and holds every token row of its slice, as float32, in
// shared memory.  All arithmetic is FP32 FMA on the CUDA cores (the work is
// tiny: 2 D r MACs per token); Q is read once from HBM/L2 straight as float32.
// The exchanges are pushed (st.async into the receiving CTA, completing bytes
// on one of its mbarriers), so every wait ends when the data has arrived rather
// than at a cluster-wide barrier:
//   1. partial y of the slice for every token (warp per column block, lane per
//      rank index, one accumulator per token), pushed to the token's owner CTA
//      (t mod 16);
//   2. the owner sums the 16 partials in CTA order, forms z = M y and pushes it
//      into every CTA;
//   3. x_out = x + Q z (thread per column, Q row in registers), bf16/fp32 store,
//      fp32 kept in shared memory; per-token partial (sum of squares, absmax)
//      of the slice, pushed into every CTA;
//   4. every CTA sums the 16 partials of every token in CTA order (the same
//      totals everywhere) and forms the row quantiser; CTA 0 writes the scales;
//   5. codes of the slice, one thread per token and group of eight columns.
// Two cluster barriers remain, both split: the first (every CTA's mbarriers
// armed before any push) around the partial projection, the last (no CTA
// leaves while its pushes may be in flight) around steps 4 and 5.
// The launch allows programmatic dependent launch: a call may start while the
// previous kernel of the stream still runs, stages its Q slice (one 16-byte
// load per thread and round, all in flight) and M, and waits for that kernel
// before it touches x or any output; it lets its own successor start at once.
// In a chain of layers this hides the launch and the Q read of each layer
// behind the previous one.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rsq {

using namespace sm100;

namespace {

constexpr int kDecCS = 16;        // CTAs per cluster: the hidden dimension is split 16 ways
constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxT = 32;
constexpr int kR = 32;            // rank slots (r <= 32, zero padded)
constexpr int kOwnMax = kDecMaxT / kDecCS;  // token rows owned by one CTA (t mod 16)

struct DecodeArgs {
    const float *Q;
    const float *M;
    uint8_t *codes;
    float *scales;
    int *status;
    long long T;
    int D;
    int r;
    float eps;
};

// Shared memory (floats unless noted), for T tokens and cw columns per CTA.
// Every float2 / float4 region starts on a multiple of 2 / 4 floats whatever
// T is (cw is a multiple of 8).
struct DecLayout {
    int cw, T;
    __host__ __device__ int off_q() const { return 0; }                          // cw x 32
    __host__ __device__ int off_x() const { return off_q() + cw * kR; }          // T x cw
    __host__ __device__ int off_z() const { return off_x() + T * cw; }           // T x 32 z (float4 reads)
    __host__ __device__ int off_mt() const { return off_z() + T * kR; }          // 32 x 32 M^T
    __host__ __device__ int off_prm() const { return off_mt() + kR * kR; }       // T x (inv, pre)
    __host__ __device__ int off_wp() const { return off_prm() + 2 * T; }         // warps x T x 32
    __host__ __device__ int off_yin() const { return off_wp() + kDecWarps * T * kR; }  // [source CTA][own row][32]
    __host__ __device__ int off_stin() const { return (off_yin() + kDecCS * kOwnMax * kR + 3) & ~3; }  // [source][T] float4
    __host__ __device__ int off_ys() const { return off_stin() + kDecCS * 4 * T; }  // warps x 32: owner's y
    __host__ __device__ int off_bar() const { return off_ys() + kDecWarps * kR; }  // 3 mbarriers (8 B each)
    __host__ __device__ int floats() const { return off_bar() + 3 * 2; }
    __host__ __device__ size_t bytes() const { return size_t(floats()) * 4; }
};

// Asynchronous 4-byte store into the shared memory of a CTA of this cluster,
// completing `bytes` on its mbarrier.
__device__ __forceinline__ void st_async_b32(uint32_t addr, uint32_t v, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
                 "r"(mbar)
                 : "memory");
}

template <class IO, int BITS>
__global__ void __launch_bounds__(kDecThreads, 1)
k_align_decode(const typename IO::T *__restrict__ x, typename IO::T *__restrict__ x_out, const DecodeArgs p) {
    extern __shared__ float4 dsm4[];
    float *smf = reinterpret_cast<float *>(dsm4);
    const int T = int(p.T), D = p.D, r = p.r;
    const int cw = D / kDecCS;
    const DecLayout L{cw, T};
    float *sq = smf + L.off_q();
    float *sx = smf + L.off_x();
    float *sz = smf + L.off_z();
    float *smt = smf + L.off_mt();
    float2 *sprm = reinterpret_cast<float2 *>(smf + L.off_prm());
    float *swp = smf + L.off_wp();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_ctarank();
    const int col0 = int(crank) * cw;
    constexpr bool kQuant = BITS > 0;  // BITS = 0: alignment only (x_out), no norm / codes
    constexpr int qmax = kQuant ? (1 << (BITS - 1)) - 1 : 1;
    const long long row_bytes = (long long)D * BITS / 8;
    // the next kernel of the stream may start staging its own Q and M now
    asm volatile("griddepcontrol.launch_dependents;");
    float *syin = smf + L.off_yin();
    float4 *sstin = reinterpret_cast<float4 *>(smf + L.off_stin());
    const uint32_t bar_y = smem_u32(smf + L.off_bar());  // own rows: partial y from every CTA
    const uint32_t bar_z = bar_y + 8;                      // z of every row from its owner
    const uint32_t bar_st = bar_y + 16;                    // partial statistics of every row from every CTA
    const int n_own = T > int(crank) ? (T - 1 - int(crank)) / kDecCS + 1 : 0;
    int err = 0;
    if (tid == 0) {
        mbar_init(bar_y, 1);
        mbar_init(bar_z, 1);
        mbar_init(bar_st, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_y, uint32_t(n_own * kDecCS * kR * 4));
        mbar_expect_tx(bar_z, uint32_t(T * kR * 4));
        if (kQuant) mbar_expect_tx(bar_st, uint32_t(kDecCS * T * 16));
    }
    cluster_arrive();  // #1 (waited before the first push)

    // ---- stage Q rows of the slice (zero padded to 32), M^T, and the token rows
    if (r == kR && (reinterpret_cast<uintptr_t>(p.Q) & 15u) == 0) {
        // the slice is contiguous: all of a thread's 16-byte loads in flight at once
        const float4 *q4 = reinterpret_cast<const float4 *>(p.Q + (size_t)col0 * kR);
        float4 *s4 = reinterpret_cast<float4 *>(sq);
        const int n4 = cw * kR / 4;
        for (int i0 = 0; i0 < n4; i0 += 8 * kDecThreads) {
            float4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = i0 + tid + k * kDecThreads;
                if (i < n4) v[k] = __ldg(q4 + i);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = i0 + tid + k * kDecThreads;
                if (i < n4) s4[i] = v[k];
            }
        }
    } else {
        for (int i = tid; i < cw * kR; i += kDecThreads) {
            const int c = i >> 5, j = i & 31;
            sq[i] = j < r ? __ldg(p.Q + (size_t)(col0 + c) * r + j) : 0.f;
        }
    }
    for (int i = tid; i < kR * kR; i += kDecThreads) {  // smt[k][j] = M[j][k]
        const int k = i >> 5, j = i & 31;
        smt[i] = (j < r && k < r) ? __ldg(p.M + j * r + k) : 0.f;
    }
    // x may be written by the previous kernel of the stream: wait for it (a no-op
    // unless this grid was launched early, programmatic dependent launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int e = tid; e < T * cw / 8; e += kDecThreads) {
        const int t = (e * 8) / cw, c = (e * 8) % cw;
        float v[8];
        load8(x + (size_t)t * D + col0 + c, v);
        store8(sx + t * cw + c, v);
    }
    __syncthreads();

    // ---- 1. partial y of this slice: warp w takes columns [w cw/8, (w+1) cw/8), lane j
    // the rank index, one accumulator per token (each Q entry loaded once); the
    // eight warp partials are then summed in warp order
    {
        const int cpw = cw / kDecWarps;
        const int c0 = warp * cpw;
        for (int t0 = 0; t0 < T; t0 += 8) {  // eight tokens per pass: eight accumulators
            const int nt = T - t0 < 8 ? T - t0 : 8;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float *xs = sx + t0 * cw;
            for (int c = c0; c < c0 + cpw; ++c) {
                const float qv = sq[c * kR + lane];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < nt) acc[k] = fmaf(xs[k * cw + c], qv, acc[k]);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < nt) swp[(warp * T + t0 + k) * kR + lane] = acc[k];
        }
    }
    __syncthreads();
    cluster_wait();  // #1: every CTA's barriers are armed before the first push
    // own rows of token t live in CTA t mod 16; push this slice's partial y there
    for (int i = tid; i < T * kR; i += kDecThreads) {
        float y = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) y += swp[w * T * kR + i];
        const int t = i / kR, k = i % kR;
        const uint32_t owner = uint32_t(t % kDecCS);
        const uint32_t dst = smem_u32(syin + (int(crank) * kOwnMax + t / kDecCS) * kR + k);
        if (!err) st_async_b32(mapa(dst, owner), __float_as_uint(y), mapa(bar_y, owner));
    }

    // ---- 2. owner of token t (t mod 16): y from the 16 partials in CTA order,
    // z = M y, pushed into every CTA
    for (int j = warp; j < n_own; j += kDecWarps) {
        const int t = int(crank) + kDecCS * j;
        if (!mbar_wait(bar_y, 0, err != 0)) err |= kErrMbarTimeout;
        float y = 0.f;
#pragma unroll
        for (int c = 0; c < kDecCS; ++c) y += syin[(c * kOwnMax + j) * kR + lane];
        // z = M y: y through shared memory, read back whole by every lane
        // (broadcast), four independent FMA chains
        float *ys = smf + L.off_ys() + warp * kR;
        __syncwarp();  // this warp's reads of its previous row are done
        ys[lane] = y;
        __syncwarp();
        float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k4 = 0; k4 < kR / 4; ++k4) {
            const float4 yv = reinterpret_cast<const float4 *>(ys)[k4];
            a4[0] = fmaf(smt[(4 * k4 + 0) * kR + lane], yv.x, a4[0]);
            a4[1] = fmaf(smt[(4 * k4 + 1) * kR + lane], yv.y, a4[1]);
            a4[2] = fmaf(smt[(4 * k4 + 2) * kR + lane], yv.z, a4[2]);
            a4[3] = fmaf(smt[(4 * k4 + 3) * kR + lane], yv.w, a4[3]);
        }
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        const uint32_t dz = smem_u32(sz + t * kR + lane);
#pragma unroll
        for (int c = 0; c < kDecCS; ++c)
            if (!err) st_async_b32(mapa(dz, uint32_t(c)), __float_as_uint(acc), mapa(bar_z, uint32_t(c)));
    }
    if (!mbar_wait(bar_z, 0, err != 0)) err |= kErrMbarTimeout;  // z of every token from its owner

    // ---- 3. x_out = x + Q z for this thread's columns, every token
    for (int c = tid; c < cw; c += kDecThreads) {
        float qv[kR];
#pragma unroll
        for (int j = 0; j < kR; j += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(sq + c * kR + j);
            qv[j] = f.x;
            qv[j + 1] = f.y;
            qv[j + 2] = f.z;
            qv[j + 3] = f.w;
        }
        // four tokens at a time: four independent FMA chains (z read four entries per load)
        for (int t0 = 0; t0 < T; t0 += 4) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < kR; j += 4) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (t0 + k < T) {
                        const float4 zz = *reinterpret_cast<const float4 *>(sz + (t0 + k) * kR + j);
                        acc[k] = fmaf(qv[j], zz.x, acc[k]);
                        acc[k] = fmaf(qv[j + 1], zz.y, acc[k]);
                        acc[k] = fmaf(qv[j + 2], zz.z, acc[k]);
                        acc[k] = fmaf(qv[j + 3], zz.w, acc[k]);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = t0 + k;
                if (t < T) {
                    const float v = sx[t * cw + c] + acc[k];
                    sx[t * cw + c] = v;
                    x_out[(size_t)t * D + col0 + c] = IO::from_f(v);
                }
            }
        }
    }
    __syncthreads();
    if constexpr (kQuant) {
    // per-token partial statistics of the slice (warp per token, lanes over
    // columns), pushed into every CTA
    for (int t = warp; t < T; t += kDecWarps) {
        const float *xr = sx + t * cw;
        float ss = 0.f, am = 0.f;
        for (int c = lane; c < cw; c += 32) {
            const float v = xr[c];
            ss = fmaf(v, v, ss);
            am = fmaxf(am, fabsf(v));
        }
        const double sd = warp_sum(double(ss));
        am = warp_max(am);
        if (lane < kDecCS && !err)
            st_async_v4(mapa(smem_u32(sstin + int(crank) * T + t), uint32_t(lane)), uint32_t(__double2loint(sd)),
                        uint32_t(__double2hiint(sd)), __float_as_uint(am), 0u, mapa(bar_st, uint32_t(lane)));
    }
    }
    cluster_arrive();  // #2 (waited at the end): no CTA leaves while its pushes may be in flight
    if constexpr (kQuant) {
    if (!mbar_wait(bar_st, 0, err != 0)) err |= kErrMbarTimeout;

    // ---- 4. row quantisers of every token from the 16 partials (CTA order: the
    // same totals everywhere)
    if (tid < T) {
        const int t = tid;
        double ss_t = 0.0;
        float am_t = 0.f;
#pragma unroll
        for (int c = 0; c < kDecCS; ++c) {
            const float4 sv = sstin[c * T + t];
            ss_t += __hiloint2double(__float_as_int(sv.y), __float_as_int(sv.x));
            am_t = fmaxf(am_t, sv.z);
        }
        const float ms = float(ss_t / double(D));
        const float rs = 1.0f / sqrtf(ms + p.eps);
        const RowQuant q = row_quant(am_t, qmax);
        sprm[t] = make_float2(q.inv, q.pre);
        if (crank == 0) p.scales[t] = am_t > 0.f ? (am_t * rs) / float(qmax) : 0.f;
    }
    __syncthreads();

    // ---- 5. codes: one thread per (token, group of eight columns)
    for (int pidx = tid; pidx < T * (cw / 8); pidx += kDecThreads) {
        const int t = pidx / (cw / 8), g = pidx % (cw / 8);
        float f[8];
        const float4 a0 = *reinterpret_cast<const float4 *>(sx + t * cw + 8 * g);
        const float4 a1 = *reinterpret_cast<const float4 *>(sx + t * cw + 8 * g + 4);
        f[0] = a0.x; f[1] = a0.y; f[2] = a0.z; f[3] = a0.w;
        f[4] = a1.x; f[5] = a1.y; f[6] = a1.z; f[7] = a1.w;
        const float2 pr = sprm[t];
        // |v| <= amax, so |v qmax / amax| <= qmax: no clamp is needed
        const uint32_t w = pack8_fast<BITS>(f, pr.x, pr.y, true);
        uint8_t *dst = p.codes + (size_t)t * row_bytes + (size_t)(col0 + 8 * g) * BITS / 8;
        if (BITS == 4) {
            *reinterpret_cast<uint32_t *>(dst) = w;
        } else {
            dst[0] = uint8_t(w);
            dst[1] = uint8_t(w >> 8);
            dst[2] = uint8_t(w >> 16);
        }
    }
    }
    if (__syncthreads_or(err)) drain_delay();
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (err && lane == 0) atomicOr(p.status, err);
    cluster_wait();
}

template <class IO, int BITS>
cudaError_t launch_typed(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes, float *scales,
                         long long T, int D, int r, float eps, cudaStream_t s) {
    static bool configured[64];
    static int max_clusters[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    auto kern = k_align_decode<IO, BITS>;
    const DecLayout L{D / kDecCS, int(T)};
    const DecLayout Lmax{8192 / kDecCS, kDecMaxT};
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Lmax.bytes()));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kDecCS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(kDecCS, 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = Lmax.bytes();
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return e;
        max_clusters[dev] = n;
        configured[dev] = true;
    }
    if (max_clusters[dev] < 1) return cudaErrorNotSupported;
    DecodeArgs a;
    a.Q = Q;
    a.M = M;
    a.codes = codes;
    a.scales = scales;
    a.status = device_status_word();
    if (!a.status) return cudaErrorInvalidValue;
    a.T = T;
    a.D = D;
    a.r = r;
    a.eps = eps;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kDecCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(kDecCS, 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = L.bytes();
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const typename IO::T *>(x), static_cast<typename IO::T *>(x_out),
                           a);
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace

bool align_decode_supports(int D, int r, long long T) {
    return T >= 1 && T <= kDecMaxT && D >= 2048 && D <= 8192 && D % (kDecCS * 8) == 0 && r >= 1 && r <= kR;
}

cudaError_t launch_align_decode(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                                float *scales, long long T, int D, int r, int bits, float eps, int dtype,
                                cudaStream_t s) {
    if (dtype == 0) {
        if (bits == 0) return launch_typed<F32, 0>(x, Q, M, x_out, codes, scales, T, D, r, eps, s);
        return bits == 4 ? launch_typed<F32, 4>(x, Q, M, x_out, codes, scales, T, D, r, eps, s)
                         : launch_typed<F32, 3>(x, Q, M, x_out, codes, scales, T, D, r, eps, s);
    }
    if (bits == 0) return launch_typed<BF16, 0>(x, Q, M, x_out, codes, scales, T, D, r, eps, s);
    return bits == 4 ? launch_typed<BF16, 4>(x, Q, M, x_out, codes, scales, T, D, r, eps, s)
                     : launch_typed<BF16, 3>(x, Q, M, x_out, codes, scales, T, D, r, eps, s);
}

}  // namespace rsq
