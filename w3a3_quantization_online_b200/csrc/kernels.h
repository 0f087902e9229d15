// kernels.h -- internal launchers behind the C ABI (not part of the public interface).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rsq {

// Device properties of the current device (cached per device ordinal).
int num_sms();
int max_smem_optin();

// Bump the process-wide launch counter (read by rsq_launch_count()).
void count_launch(int n = 1);

// Generic CUDA-core path: any supported D, r, dtype.  quant=false computes
// x_out only (codes / scales ignored).
cudaError_t launch_align_generic(const void *x, const float *Q, const float *M, void *x_out,
                                 uint8_t *codes, float *scales, int64_t T, int D, int r,
                                 int bits, float eps, int dtype, bool quant, cudaStream_t s);

// Generic randomised Hadamard + quantiser: m in {1, 12}, any supported d.
cudaError_t launch_rht_generic(const void *x, const int8_t *signs, int m, uint8_t *codes,
                               float *scales, int64_t T, int d, int bits, int dtype,
                               cudaStream_t s);

// Device-side status word of the current device (bits from sm100::kErr*), or
// nullptr if its address cannot be obtained.
int *device_status_word();
// Device word that rsq_device_status() takes the status into (same device).
int *status_taken_word();

// Tensor-core alignment + RMSNorm + quantiser (bf16, D in {4096, 8192}, r <= 32).
bool align_tc_supports(int D, int r, int dtype, long long T);
// *launched is false (and cudaSuccess returned) when the cluster shape cannot be
// scheduled on this device; the caller then uses the generic kernel.
cudaError_t launch_align_tc(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                            float *scales, long long T, int D, int r, int bits, float eps, cudaStream_t s,
                            bool *launched);

// Tensor-core alignment + RMSNorm + quantiser with two 64-row tiles in flight
// per CTA (bf16, D in {4096, 8192}, r <= 32); same contract as launch_align_tc.
// Decode-size alignment + RMSNorm + quantiser: one cluster of 16 CTAs, FP32 FMAs
// (T <= 32, 2048 <= D <= 8192, D % 128 == 0, r <= 32, bf16 or fp32 I/O).
// Returns cudaErrorNotSupported if the cluster cannot be co-scheduled.
bool align_decode_supports(int D, int r, long long T);
cudaError_t launch_align_decode(const void *x, const float *Q, const float *M, void *x_out, uint8_t *codes,
                                float *scales, long long T, int D, int r, int bits, float eps, int dtype,
                                cudaStream_t s);

// The generic kernel with the input formed as SiLU(a) * b in fp32.
cudaError_t launch_rht_gate_generic(const void *a, const void *b, const int8_t *signs, int m, uint8_t *codes,
                                    float *scales, int64_t T, int d, int bits, int dtype, cudaStream_t s);

// Randomised Hadamard H_1024 (x) H_12 of order 12288 (Paley H_12), bf16, INT4, with
// the H_128 stage of H_1024 on the tensor cores.
bool rht_kron_tc_supports(int d, int m, int dtype, int bits, long long T);
cudaError_t launch_rht_kron_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                               cudaStream_t s);
// The gated down_proj input SiLU(a) * b (fp32) through the same transform on the CUDA cores.
bool rht_kron_gate_supports(int d, int m, int dtype, int bits, long long T);
cudaError_t launch_rht_kron_gate(const void *a, const void *b, const int8_t *signs, uint8_t *codes, float *scales,
                                 long long T, cudaStream_t s);

// Attention: per-head randomised Hadamard (I (x) H_dh), rotation only (x_out)
// or with per-(token, head) quantisation (quant), and head mixing (H_nh (x) I)
// with per-token quantisation.  signs may be nullptr (all +1).
bool head_rht_supports(int d, int n_heads);
bool head_mix_supports(int d, int n_heads);
cudaError_t launch_head_rht(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales,
                            long long T, int d, int n_heads, int bits, bool quant, int dtype, cudaStream_t s);
cudaError_t launch_head_mix(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T, int d,
                            int n_heads, int bits, int dtype, cudaStream_t s);
// Head mixing + per-token quantiser on the tensor cores (bf16, 32 heads of 128).
bool head_mix_tc_supports(int d, int n_heads, int dtype, long long T);
cudaError_t launch_head_mix_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T,
                               int bits, cudaStream_t s);
// The same per-head rotation / quantisation on the tensor cores (bf16, d_h in {64, 128}).
bool head_tc_supports(int d, int n_heads, int dtype, long long T);
cudaError_t launch_head_tc(const void *x, const int8_t *signs, void *x_out, uint8_t *codes, float *scales,
                           long long T, int d, int n_heads, int bits, bool quant, cudaStream_t s);

// INT4 consumer GEMM: y = round16(float(codes_a codes_w^T) * sa[t] * sw[n]),
// fp16 (out_f16) or bf16 out, optional raw int32 accumulators.
bool w4a4_gemm_supports(long long T, int N, int K);
// w: packed weight codes (N x K/2), or with w_prepared the int8 weights (N x K)
// written by launch_w4a4_unpack_weights.
cudaError_t launch_w4a4_gemm(const uint8_t *codes_a, const float *sa, const void *w, bool w_prepared, const float *sw,
                             void *y, int32_t *acc, long long T, int N, int K, int out_f16, cudaStream_t s);
cudaError_t launch_w4a4_unpack_weights(const uint8_t *codes_w, int8_t *w_s8, int N, int K, cudaStream_t s);

// Offline (Q, M) construction from two rotations; workspace from the caller.
bool qm_supports(int D, int r);
size_t qm_workspace_bytes(int D, int r);
cudaError_t launch_qm_build(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M,
                            void *workspace, cudaStream_t s);
// The library's own fixed scratch array for the construction (size, and its
// device address on the current device: obtained once per device).
size_t qm_static_scratch_bytes();
cudaError_t qm_static_scratch(void **ptr);

// Randomised Hadamard of order 4096 or 8192 with the first stage on tcgen05
// (m = 1, bf16, INT4/INT3).
bool rht_tc_supports(int d, int m, int dtype, int bits, long long T);
cudaError_t launch_rht_tc(const void *x, const int8_t *signs, uint8_t *codes, float *scales, long long T, int d,
                          int bits, cudaStream_t s);

// FlatQuant's Kronecker affine transform vec(P1^T X P2) + per-token quantiser,
// float64 products on the CUDA cores: n1, n2 multiples of 4 in [4, 128],
// n1 n2 <= 4096.
bool kron_affine_supports(int n1, int n2);
cudaError_t launch_kron_affine_quant(const void *x, const float *P1, const float *P2, int n1, int n2,
                                     uint8_t *codes, float *scales, long long T, int bits, int dtype,
                                     cudaStream_t s);

}  // namespace rsq
