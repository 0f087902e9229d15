// rsq_abi.cu -- the extern "C" entry points declared in include/rsq.h.
//
// Every argument is checked on the host before anything is enqueued; a
// rejected call returns a status and touches no memory.  The entry points then
// pick a kernel by shape and dtype and enqueue it on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "kernels.h"
#include "rsq.h"
#include "sm100.cuh"

namespace rsq {

// Device-side status word: kernels OR error bits into it (bounded waits that
// timed out); rsq_device_status() takes it (atomic exchange with 0) into
// g_status_taken on the caller's stream and copies that to the host.
__device__ int g_device_status;
__device__ int g_status_taken;

namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_align_kernel{0};  // 0 auto, 1 generic, 2 cluster tensor core, 4 decode
std::atomic<int> g_rht_kernel{0};    // 0 auto, 1 generic, 3 tensor core, 4 Kronecker 12288
thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
int g_smem[kMaxDevices];

int cur_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    return dev;
}
}  // namespace

void count_launch(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }

namespace {
// One thread waits, through the same bounded wait the kernels use, on an
// mbarrier that nothing arrives on: the wait gives up after limit_ns and the
// timeout bit goes into the device status word; the kernel then returns.
__global__ void k_selftest_wait(int *status, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = sm100::smem_u32(&bar);
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
    if (!sm100::mbar_wait(b, 0u, false, limit_ns)) atomicOr(status, sm100::kErrMbarTimeout);
}

// Takes the status word in one atomic step, so that a bit a kernel on another
// stream sets at the same moment is either taken now or left for the next call.
__global__ void k_take_status(int *word, int *out) { *out = atomicExch(word, 0); }
}  // namespace

int *status_taken_word() {
    static int *addr[kMaxDevices];
    const int dev = cur_device();
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_taken) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int *>(p);
    }
    return addr[dev];
}

int num_sms() {
    const int dev = cur_device();
    if (g_sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        g_sms[dev] = v;
    }
    return g_sms[dev];
}

int *device_status_word() {
    static int *addr[kMaxDevices];
    const int dev = cur_device();
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int *>(p);
    }
    return addr[dev];
}

int max_smem_optin() {
    const int dev = cur_device();
    if (g_smem[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || v <= 0)
            v = 227 * 1024;
        g_smem[dev] = v;
    }
    return g_smem[dev];
}

}  // namespace rsq

namespace {

using rsq::g_last_cuda_error;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
};

Span span(const void *p, uint64_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Span{a, a + uintptr_t(bytes)};
}

bool overlap(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi; }

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int finish(cudaError_t e) {
    if (e != cudaSuccess) {
        g_last_cuda_error = int(e);
        return RSQ_ERR_CUDA;
    }
    return RSQ_OK;
}

int elem_bytes(int dtype) { return dtype == RSQ_F32 ? 4 : 2; }

// Shared checks of the alignment entry points.
int check_align_args(const void *x, const float *Q, const float *M, const void *x_out, int64_t T,
                     int D, int r, int dtype) {
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (T < 0 || D < 16 || D > 32768 || D % 16 != 0 || r < 1 || r > 64) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !Q || !M || !x_out) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(Q) || !aligned16(M) || !aligned16(x_out)) return RSQ_ERR_ALIGN;
    const uint64_t act = uint64_t(T) * uint64_t(D) * uint64_t(elem_bytes(dtype));
    const Span sx = span(x, act), so = span(x_out, act);
    const Span sq = span(Q, uint64_t(D) * r * 4), sm = span(M, uint64_t(r) * r * 4);
    if (x != x_out && overlap(sx, so)) return RSQ_ERR_ALIAS;
    if (overlap(so, sq) || overlap(so, sm)) return RSQ_ERR_ALIAS;
    return RSQ_OK;
}

}  // namespace

extern "C" {

int rsq_residual_align(const void *x, const float *Q, const float *M, void *x_out, int64_t T,
                       int D, int r, int dtype, void *stream) {
    int st = check_align_args(x, Q, M, x_out, T, D, r, dtype);
    if (st != RSQ_OK || T == 0) return st;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // the kernels of rsq_align_norm_quant instantiated without the norm and the
    // codes (bits = 0), chosen the same way
    const int which = rsq::g_align_kernel.load(std::memory_order_relaxed);
    if (((which == 0 && T <= 16) || which == 4) && rsq::align_decode_supports(D, r, T)) {
        const cudaError_t e = rsq::launch_align_decode(x, Q, M, x_out, nullptr, nullptr, T, D, r, 0, 0.f, dtype, cs);
        if (e != cudaErrorNotSupported) return finish(e);
    }
    if ((which == 0 || which == 2) && rsq::align_tc_supports(D, r, dtype, T)) {
        bool launched = false;
        const cudaError_t e = rsq::launch_align_tc(x, Q, M, x_out, nullptr, nullptr, T, D, r, 0, 0.f, cs, &launched);
        if (e != cudaSuccess) return finish(e);
        if (launched) return RSQ_OK;
    }
    if (which >= 2) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_align_generic(x, Q, M, x_out, nullptr, nullptr, T, D, r, 4, 0.f, dtype, false, cs));
}

int rsq_align_norm_quant(const void *x, const float *Q, const float *M, void *x_out,
                         uint8_t *codes, float *scales, int64_t T, int D, int r, int bits,
                         float eps, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    int st = check_align_args(x, Q, M, x_out, T, D, r, dtype);
    if (st != RSQ_OK) return st;
    if (!std::isfinite(eps) || eps < 0.f) return RSQ_ERR_VALUE;
    if (T == 0) return RSQ_OK;
    if (!codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales)) return RSQ_ERR_ALIGN;
    const uint64_t act = uint64_t(T) * uint64_t(D) * uint64_t(elem_bytes(dtype));
    const Span sx = span(x, act), so = span(x_out, act);
    const Span sc = span(codes, uint64_t(T) * uint64_t(D) * bits / 8), ss = span(scales, uint64_t(T) * 4);
    if (overlap(sc, sx) || overlap(sc, so) || overlap(ss, sx) || overlap(ss, so) || overlap(sc, ss) ||
        overlap(sc, span(Q, uint64_t(D) * r * 4)) || overlap(ss, span(Q, uint64_t(D) * r * 4)) ||
        overlap(sc, span(M, uint64_t(r) * r * 4)) || overlap(ss, span(M, uint64_t(r) * r * 4)))
        return RSQ_ERR_ALIAS;
    const int which = rsq::g_align_kernel.load(std::memory_order_relaxed);
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // decode kernel: chosen automatically up to 16 rows (measured: beyond that the
    // tensor-core kernel's flat ~16 us per call is shorter), on request up to 32
    if (((which == 0 && T <= 16) || which == 4) && rsq::align_decode_supports(D, r, T)) {
        const cudaError_t e = rsq::launch_align_decode(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, dtype, cs);
        if (e != cudaErrorNotSupported) return finish(e);  // not co-schedulable: another kernel serves it
    }
    if ((which == 0 || which == 2) && rsq::align_tc_supports(D, r, dtype, T)) {
        bool launched = false;
        const cudaError_t e = rsq::launch_align_tc(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, cs, &launched);
        if (e != cudaSuccess) return finish(e);
        if (launched) return RSQ_OK;
    }
    if (which == 2 || which == 4) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_align_generic(x, Q, M, x_out, codes, scales, T, D, r, bits, eps, dtype,
                                            true, static_cast<cudaStream_t>(stream)));
}

int rht_quant(const void *x, const int8_t *signs, int m, uint8_t *codes, float *scales, int64_t T,
              int d, int bits, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (m != 1 && m != 12) return RSQ_ERR_UNSUPPORTED;
    if (T < 0 || d < 16 || d > 32768 || d % 16 != 0 || d % m != 0) return RSQ_ERR_SHAPE;
    const int n2 = d / m;
    if (!is_pow2(n2) || n2 < 16 || n2 > 16384) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !signs || !codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(signs) || !aligned16(codes) || !aligned16(scales)) return RSQ_ERR_ALIGN;
    const Span sx = span(x, uint64_t(T) * d * elem_bytes(dtype)), sg = span(signs, uint64_t(d));
    const Span sc = span(codes, uint64_t(T) * d * bits / 8), ss = span(scales, uint64_t(T) * 4);
    if (overlap(sc, sx) || overlap(sc, sg) || overlap(sc, ss) || overlap(ss, sx) || overlap(ss, sg))
        return RSQ_ERR_ALIAS;
    const int which = rsq::g_rht_kernel.load(std::memory_order_relaxed);
    if ((which == 0 || which == 3) && rsq::rht_tc_supports(d, m, dtype, bits, T))
        return finish(rsq::launch_rht_tc(x, signs, codes, scales, T, d, bits, static_cast<cudaStream_t>(stream)));
    if ((which == 0 || which == 4) && rsq::rht_kron_tc_supports(d, m, dtype, bits, T))
        return finish(rsq::launch_rht_kron_tc(x, signs, codes, scales, T, static_cast<cudaStream_t>(stream)));
    if (which == 3 || which == 4) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_rht_generic(x, signs, m, codes, scales, T, d, bits, dtype,
                                          static_cast<cudaStream_t>(stream)));
}

int rht_quant_silu_gate(const void *a, const void *b, const int8_t *signs, int m, uint8_t *codes, float *scales,
                        int64_t T, int d, int bits, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (m != 1 && m != 12) return RSQ_ERR_UNSUPPORTED;
    if (T < 0 || d < 16 || d > 32768 || d % 16 != 0 || d % m != 0) return RSQ_ERR_SHAPE;
    const int n2 = d / m;
    if (!is_pow2(n2) || n2 < 16 || n2 > 16384) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!a || !b || !signs || !codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(a) || !aligned16(b) || !aligned16(signs) || !aligned16(codes) || !aligned16(scales))
        return RSQ_ERR_ALIGN;
    const uint64_t in_bytes = uint64_t(T) * d * elem_bytes(dtype);
    const Span sa = span(a, in_bytes), sb = span(b, in_bytes), sg = span(signs, uint64_t(d));
    const Span sc = span(codes, uint64_t(T) * d * bits / 8), ss = span(scales, uint64_t(T) * 4);
    // the inputs may overlap each other (read only); no output may overlap anything
    if (overlap(sc, sa) || overlap(sc, sb) || overlap(sc, sg) || overlap(sc, ss) || overlap(ss, sa) ||
        overlap(ss, sb) || overlap(ss, sg))
        return RSQ_ERR_ALIAS;
    const int which = rsq::g_rht_kernel.load(std::memory_order_relaxed);
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((which == 0 || which == 4) && rsq::rht_kron_gate_supports(d, m, dtype, bits, T))
        return finish(rsq::launch_rht_kron_gate(a, b, signs, codes, scales, T, cs));
    if (which == 3 || which == 4) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_rht_gate_generic(a, b, signs, m, codes, scales, T, d, bits, dtype, cs));
}

int rht_heads(const void *x, const int8_t *signs, int n_heads, void *x_out, int64_t T, int d, int dtype,
              void *stream) {
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (T < 0 || d < 16 || d > 32768 || !rsq::head_rht_supports(d, n_heads)) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !x_out) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(x_out) || (signs && !aligned16(signs))) return RSQ_ERR_ALIGN;
    const uint64_t bytes = uint64_t(T) * d * elem_bytes(dtype);
    const Span sx = span(x, bytes), so = span(x_out, bytes);
    if (x != x_out && overlap(sx, so)) return RSQ_ERR_ALIAS;
    if (signs && overlap(so, span(signs, uint64_t(d)))) return RSQ_ERR_ALIAS;
    const int which = rsq::g_rht_kernel.load(std::memory_order_relaxed);
    if (which != 1 && rsq::head_tc_supports(d, n_heads, dtype, T))
        return finish(rsq::launch_head_tc(x, signs, x_out, nullptr, nullptr, T, d, n_heads, 4, false,
                                          static_cast<cudaStream_t>(stream)));
    if (which == 3) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_head_rht(x, signs, x_out, nullptr, nullptr, T, d, n_heads, 4, false, dtype,
                                       static_cast<cudaStream_t>(stream)));
}

int rht_heads_quant(const void *x, const int8_t *signs, int n_heads, uint8_t *codes, float *scales, int64_t T,
                    int d, int bits, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (T < 0 || d < 16 || d > 32768 || !rsq::head_rht_supports(d, n_heads)) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (signs && !aligned16(signs)))
        return RSQ_ERR_ALIGN;
    const Span sx = span(x, uint64_t(T) * d * elem_bytes(dtype));
    const Span sc = span(codes, uint64_t(T) * d * bits / 8), ss = span(scales, uint64_t(T) * n_heads * 4);
    if (overlap(sc, sx) || overlap(ss, sx) || overlap(sc, ss)) return RSQ_ERR_ALIAS;
    if (signs) {
        const Span sg = span(signs, uint64_t(d));
        if (overlap(sc, sg) || overlap(ss, sg)) return RSQ_ERR_ALIAS;
    }
    const int which = rsq::g_rht_kernel.load(std::memory_order_relaxed);
    if (which != 1 && rsq::head_tc_supports(d, n_heads, dtype, T))
        return finish(rsq::launch_head_tc(x, signs, nullptr, codes, scales, T, d, n_heads, bits, true,
                                          static_cast<cudaStream_t>(stream)));
    if (which == 3) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_head_rht(x, signs, nullptr, codes, scales, T, d, n_heads, bits, true, dtype,
                                       static_cast<cudaStream_t>(stream)));
}

int rht_head_mix_quant(const void *x, const int8_t *signs, int n_heads, uint8_t *codes, float *scales, int64_t T,
                       int d, int bits, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (T < 0 || d < 16 || d > 32768 || d % 16 != 0 || !rsq::head_mix_supports(d, n_heads)) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (signs && !aligned16(signs)))
        return RSQ_ERR_ALIGN;
    const Span sx = span(x, uint64_t(T) * d * elem_bytes(dtype));
    const Span sc = span(codes, uint64_t(T) * d * bits / 8), ss = span(scales, uint64_t(T) * 4);
    if (overlap(sc, sx) || overlap(ss, sx) || overlap(sc, ss)) return RSQ_ERR_ALIAS;
    if (signs) {
        const Span sg = span(signs, uint64_t(d));
        if (overlap(sc, sg) || overlap(ss, sg)) return RSQ_ERR_ALIAS;
    }
    const int which = rsq::g_rht_kernel.load(std::memory_order_relaxed);
    if (which != 1 && rsq::head_mix_tc_supports(d, n_heads, dtype, T))
        return finish(rsq::launch_head_mix_tc(x, signs, codes, scales, T, bits, static_cast<cudaStream_t>(stream)));
    if (which == 3) return RSQ_ERR_UNSUPPORTED;
    return finish(rsq::launch_head_mix(x, signs, codes, scales, T, d, n_heads, bits, dtype,
                                       static_cast<cudaStream_t>(stream)));
}

int kron_affine_quant(const void *x, const float *P1, const float *P2, int n1, int n2, uint8_t *codes,
                      float *scales, int64_t T, int bits, int dtype, void *stream) {
    if (bits != 3 && bits != 4) return RSQ_ERR_BITS;
    if (dtype != RSQ_F32 && dtype != RSQ_BF16) return RSQ_ERR_DTYPE;
    if (T < 0 || !rsq::kron_affine_supports(n1, n2)) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!x || !P1 || !P2 || !codes || !scales) return RSQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(P1) || !aligned16(P2) || !aligned16(codes) || !aligned16(scales))
        return RSQ_ERR_ALIGN;
    const int64_t d = int64_t(n1) * n2;
    const Span sx = span(x, uint64_t(T) * d * elem_bytes(dtype));
    const Span s1 = span(P1, uint64_t(n1) * n1 * 4), s2 = span(P2, uint64_t(n2) * n2 * 4);
    const Span sc = span(codes, uint64_t(T) * d * bits / 8), ss = span(scales, uint64_t(T) * 4);
    const Span ins[3] = {sx, s1, s2};
    for (int i = 0; i < 3; ++i)
        if (overlap(sc, ins[i]) || overlap(ss, ins[i])) return RSQ_ERR_ALIAS;
    if (overlap(sc, ss)) return RSQ_ERR_ALIAS;
    return finish(rsq::launch_kron_affine_quant(x, P1, P2, n1, n2, codes, scales, T, bits, dtype,
                                                static_cast<cudaStream_t>(stream)));
}

// Shared checks and launch of the two GEMM entry points: w is the packed weight
// codes (N x K/2 bytes) or, with w_prepared, the int8 weights (N x K bytes).
static int w4a4_gemm_common(const uint8_t *codes_a, const float *scales_a, const void *w, bool w_prepared,
                            const float *scales_w, void *y, int32_t *acc, int64_t T, int N, int K, int out_dtype,
                            void *stream) {
    if (out_dtype != RSQ_BF16 && out_dtype != RSQ_F16) return RSQ_ERR_DTYPE;
    if (T < 0 || N < 8 || N % 8 != 0 || N > 65536 || K < 128 || K % 128 != 0 || K > 65536) return RSQ_ERR_SHAPE;
    if (T == 0) return RSQ_OK;
    if (!rsq::w4a4_gemm_supports(T, N, K)) return RSQ_ERR_SHAPE;
    if (!codes_a || !scales_a || !w || !scales_w || !y) return RSQ_ERR_NULL;
    if (!aligned16(codes_a) || !aligned16(scales_a) || !aligned16(w) || !aligned16(scales_w) || !aligned16(y) ||
        (acc && !aligned16(acc)))
        return RSQ_ERR_ALIGN;
    const uint64_t w_bytes = uint64_t(N) * (w_prepared ? K : K / 2);
    const Span in[4] = {span(codes_a, uint64_t(T) * (K / 2)), span(scales_a, uint64_t(T) * 4), span(w, w_bytes),
                        span(scales_w, uint64_t(N) * 4)};
    const Span sy = span(y, uint64_t(T) * N * 2);
    for (const Span &i : in)
        if (overlap(sy, i)) return RSQ_ERR_ALIAS;
    if (acc) {
        const Span sacc = span(acc, uint64_t(T) * N * 4);
        if (overlap(sacc, sy)) return RSQ_ERR_ALIAS;
        for (const Span &i : in)
            if (overlap(sacc, i)) return RSQ_ERR_ALIAS;
    }
    return finish(rsq::launch_w4a4_gemm(codes_a, scales_a, w, w_prepared, scales_w, y, acc, T, N, K,
                                        out_dtype == RSQ_F16, static_cast<cudaStream_t>(stream)));
}

int w4a4_gemm(const uint8_t *codes_a, const float *scales_a, const uint8_t *codes_w, const float *scales_w, void *y,
              int32_t *acc, int64_t T, int N, int K, int out_dtype, void *stream) {
    return w4a4_gemm_common(codes_a, scales_a, codes_w, false, scales_w, y, acc, T, N, K, out_dtype, stream);
}

int w4a4_prepare_weights(const uint8_t *codes_w, int N, int K, int8_t *w_s8, void *stream) {
    if (N < 8 || N % 8 != 0 || N > 65536 || K < 128 || K % 128 != 0 || K > 65536) return RSQ_ERR_SHAPE;
    if (!codes_w || !w_s8) return RSQ_ERR_NULL;
    if (!aligned16(codes_w) || !aligned16(w_s8)) return RSQ_ERR_ALIGN;
    if (overlap(span(codes_w, uint64_t(N) * (K / 2)), span(w_s8, uint64_t(N) * K))) return RSQ_ERR_ALIAS;
    return finish(rsq::launch_w4a4_unpack_weights(codes_w, w_s8, N, K, static_cast<cudaStream_t>(stream)));
}

int w4a4_gemm_s8w(const uint8_t *codes_a, const float *scales_a, const int8_t *w_s8, const float *scales_w, void *y,
                  int32_t *acc, int64_t T, int N, int K, int out_dtype, void *stream) {
    return w4a4_gemm_common(codes_a, scales_a, w_s8, true, scales_w, y, acc, T, N, K, out_dtype, stream);
}

uint64_t rsq_qm_workspace_bytes(int D, int r) {
    if (!rsq::qm_supports(D, r)) return 0;
    return uint64_t(rsq::qm_workspace_bytes(D, r));
}

int rsq_qm_build(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M, void *workspace,
                 uint64_t workspace_bytes, void *stream) {
    if (!rsq::qm_supports(D, r)) return RSQ_ERR_SHAPE;
    if (iters < 1 || iters > 1000) return RSQ_ERR_VALUE;
    if (!R_in || !R_out || !Q || !M || !workspace) return RSQ_ERR_NULL;
    if (!aligned16(R_in) || !aligned16(R_out) || !aligned16(Q) || !aligned16(M) || !aligned16(workspace))
        return RSQ_ERR_ALIGN;
    const uint64_t need = uint64_t(rsq::qm_workspace_bytes(D, r));
    if (workspace_bytes < need) return RSQ_ERR_VALUE;
    const Span rin = span(R_in, uint64_t(D) * D * 4), rout = span(R_out, uint64_t(D) * D * 4);
    const Span sq = span(Q, uint64_t(D) * r * 4), sm = span(M, uint64_t(r) * r * 4), sw = span(workspace, need);
    const Span outs[3] = {sq, sm, sw};
    for (int i = 0; i < 3; ++i) {
        if (overlap(outs[i], rin) || overlap(outs[i], rout)) return RSQ_ERR_ALIAS;
        for (int j = i + 1; j < 3; ++j)
            if (overlap(outs[i], outs[j])) return RSQ_ERR_ALIAS;
    }
    return finish(rsq::launch_qm_build(R_in, R_out, D, r, iters, Q, M, workspace, static_cast<cudaStream_t>(stream)));
}

int rsq_qm_build_fixed_scratch(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M,
                               void *stream) {
    if (!rsq::qm_supports(D, r)) return RSQ_ERR_SHAPE;
    if (rsq::qm_workspace_bytes(D, r) > rsq::qm_static_scratch_bytes()) return RSQ_ERR_SHAPE;
    if (iters < 1 || iters > 1000) return RSQ_ERR_VALUE;
    if (!R_in || !R_out || !Q || !M) return RSQ_ERR_NULL;
    if (!aligned16(R_in) || !aligned16(R_out) || !aligned16(Q) || !aligned16(M)) return RSQ_ERR_ALIGN;
    const Span rin = span(R_in, uint64_t(D) * D * 4), rout = span(R_out, uint64_t(D) * D * 4);
    const Span sq = span(Q, uint64_t(D) * r * 4), sm = span(M, uint64_t(r) * r * 4);
    if (overlap(sq, rin) || overlap(sq, rout) || overlap(sm, rin) || overlap(sm, rout) || overlap(sq, sm))
        return RSQ_ERR_ALIAS;
    void *scratch = nullptr;
    const cudaError_t e = rsq::qm_static_scratch(&scratch);
    if (e != cudaSuccess) return finish(e);
    return finish(rsq::launch_qm_build(R_in, R_out, D, r, iters, Q, M, scratch, static_cast<cudaStream_t>(stream)));
}

const char *rsq_status_string(int status) {
    switch (status) {
        case RSQ_OK: return "RSQ_OK";
        case RSQ_ERR_NULL: return "RSQ_ERR_NULL: a required pointer is NULL";
        case RSQ_ERR_SHAPE: return "RSQ_ERR_SHAPE: unsupported or invalid shape";
        case RSQ_ERR_DTYPE: return "RSQ_ERR_DTYPE: dtype must be RSQ_F32 or RSQ_BF16";
        case RSQ_ERR_BITS: return "RSQ_ERR_BITS: bits must be 3 or 4";
        case RSQ_ERR_ALIGN: return "RSQ_ERR_ALIGN: pointers must be 16-byte aligned";
        case RSQ_ERR_ALIAS: return "RSQ_ERR_ALIAS: buffers overlap (only x_out == x is allowed)";
        case RSQ_ERR_UNSUPPORTED: return "RSQ_ERR_UNSUPPORTED: configuration not built";
        case RSQ_ERR_CUDA: return "RSQ_ERR_CUDA: a CUDA call failed (see rsq_last_cuda_error)";
        case RSQ_ERR_VALUE: return "RSQ_ERR_VALUE: a scalar argument is out of range";
        default: return "unknown rsq status";
    }
}

int rsq_last_cuda_error(void) { return g_last_cuda_error; }

int rsq_select_align_kernel(int which) {
    if (which < 0 || which > 4 || which == 3) return -1;
    return rsq::g_align_kernel.exchange(which);
}

int rsq_select_rht_kernel(int which) {
    if (which < 0 || which > 4 || which == 2) return -1;
    return rsq::g_rht_kernel.exchange(which);
}

int rsq_device_status(void *stream, int *status) {
    if (!status) return RSQ_ERR_NULL;
    int *word = rsq::device_status_word();
    int *taken = rsq::status_taken_word();
    if (!word || !taken) return finish(cudaErrorInvalidDevice);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rsq::k_take_status<<<1, 1, 0, s>>>(word, taken);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) rsq::count_launch(1);
    int v = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, taken, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) *status = v;
    return finish(e);
}

uint64_t rsq_launch_count(void) { return rsq::g_launches.load(std::memory_order_relaxed); }

int rsq_selftest_wait_timeout(int limit_ms, void *stream) {
    if (limit_ms < 1 || limit_ms > 1000) return RSQ_ERR_VALUE;
    int *word = rsq::device_status_word();
    if (!word) return finish(cudaErrorInvalidDevice);
    rsq::k_selftest_wait<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(word, (unsigned long long)limit_ms * 1000000ull);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) rsq::count_launch(1);
    return finish(e);
}

}  // extern "C"
