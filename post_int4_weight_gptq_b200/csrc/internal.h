// Internal launchers shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace piq {

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  int sm_count = 0;
  int major = 0;
  int minor = 0;
};
int device_info(DeviceInfo* out);  // PIQ_OK / PIQ_ERR_CUDA / PIQ_ERR_UNSUPPORTED_DEVICE

// Count one kernel launch (piq_kernel_launches).
void note_launch(int count = 1);

// Host-side fault injection for testing callers' error handling: with the
// environment variable PIQ_FAULT set to notpd, timeout or oom, every compute
// entry point returns PIQ_ERR_NOT_PD, PIQ_ERR_TIMEOUT or PIQ_ERR_CUDA (recorded
// as cudaErrorMemoryAllocation) after checking its arguments and before any
// device work; unset or any other value: PIQ_OK.
int injected_fault();

// PIQ_OK for cudaSuccess, else PIQ_ERR_CUDA with the error recorded for
// piq_last_cuda_error.
int cuda_rc(cudaError_t e);
// Copy the status word back, synchronize `stream` and return the status code
// (PIQ_ERR_CUDA, recorded, when the copy or a kernel of the call failed).
// host_st, when given, receives the whole status word.
int finish_call(DeviceStatus* st, cudaStream_t stream, DeviceStatus* host_st);

// ------------------------------------------------------ tensor-core GEMMs (tc_gemm.cu)
// H (+)= X^T X: upper-triangle tiles of a [in, in] fp32 matrix (row-major).
int launch_syrk_xtx(const uint16_t* X, int64_t n, int64_t in, float* H, int accumulate,
                    DeviceStatus* st, cudaStream_t stream);
// Fused ||X D_b^T||_F^2 for b < batch, D stacked [batch][rows][in] bf16.
// Writes four doubles per output tile into `partials` (size: sumsq_partials_count).
int launch_err_sumsq(const uint16_t* X, int64_t n, int64_t in, const uint16_t* D, int64_t rows,
                     int batch, double* partials, DeviceStatus* st, cudaStream_t stream);
int64_t sumsq_partials_count(int64_t n, int64_t rows, int batch);
// Fixed-order sum of the partials of each batch entry into out[batch].
int launch_reduce_partials(const double* partials, int64_t n, int64_t rows, int batch,
                           double* out, cudaStream_t stream);
// out[b] = fixed-order sum of partials[b * per .. (b + 1) * per).
int launch_reduce_sum(const double* partials, int64_t per, int batch, double* out,
                      cudaStream_t stream);

// E = 2 sum_r D_r Hu D_r^T from bf16 hi/lo pairs (tc_gemm.cu): D_hi, D_lo [out][in],
// Hu_hi, Hu_lo [in][in] (Hu = upper triangle of H, diagonal halved), D fp32 [out][in].
// Writes err_dot_partials_count(out, in) doubles.
int launch_err_dot(const uint16_t* D_hi, const uint16_t* D_lo, const uint16_t* Hu_hi,
                   const uint16_t* Hu_lo, const float* D, int64_t out, int64_t in,
                   double* partials, DeviceStatus* st, cudaStream_t stream);
int64_t err_dot_partials_count(int64_t out, int64_t in);

// ------------------------------------------ output error through H (errh.cu)
// err = ||X D^T||_F^2 = 2 sum_r D_r Hu D_r^T with D [out, in] fp32 and H = X^T X
// (upper triangle read).  Scratch: dsplit 2 out in, hsplit 2 in in bf16;
// partials err_via_h_partials(out, in) doubles.
int run_error_via_h(const float* D, int64_t out, int64_t in, const float* H, uint16_t* dsplit,
                    uint16_t* hsplit, double* partials, double* err, DeviceStatus* st,
                    cudaStream_t stream);
int64_t err_via_h_partials(int64_t out, int64_t in);

// ------------------------------------------------------ FP32 SIMT GEMM (simt_gemm.cu)
// C = alpha * A * op(B) + beta * C, row-major; op(B) = B or B^T (trans_b).
// mode 0: plain; 1: only tiles touching the lower triangle of C (M == N);
// 2: A lower triangular (entries right of the diagonal are skipped per row tile);
// 3: op(B)[k][n] = 0 for k > n (k stops at the column tile's end);
// 4: op(B)[k][n] = 0 for k < n (k starts at the column tile's start).
// Batching over blockIdx.z: entry z uses A + z*stride_a (and B, C alike); with
// m_total > 0 entry z has min(M, m_total - z*m_step) rows, and K the same when
// k_follows_m (a square triangular A).
struct GemmBatch {
  int count = 1;
  int64_t stride_a = 0, stride_b = 0, stride_c = 0;
  int64_t m_total = 0, m_step = 0;
  bool k_follows_m = false;
};
int launch_simt_gemm(int M, int N, int K, float alpha, const float* A, int64_t lda,
                     const float* B, int64_t ldb, bool trans_b, float beta, float* C,
                     int64_t ldc, int mode, const DeviceStatus* st, cudaStream_t stream,
                     const GemmBatch& bt = GemmBatch());

// ------------------------------------------- FP32-accurate tensor-core GEMM (tc_sgemm.cu)
// Same contract as launch_simt_gemm, on tcgen05 (three TF32 passes).  Returns
// PIQ_ERR_INVALID_ARG when an operand is not TMA-compatible (16-byte aligned
// base and row stride); launch_gemm_f32 then falls back to the SIMT kernel.
int launch_tc_sgemm(int M, int N, int K, float alpha, const float* A, int64_t lda,
                    const float* B, int64_t ldb, bool trans_b, float beta, float* C, int64_t ldc,
                    int mode, DeviceStatus* st, cudaStream_t stream,
                    const GemmBatch& bt = GemmBatch());
int launch_gemm_f32(int M, int N, int K, float alpha, const float* A, int64_t lda, const float* B,
                    int64_t ldb, bool trans_b, float beta, float* C, int64_t ldc, int mode,
                    DeviceStatus* st, cudaStream_t stream, const GemmBatch& bt = GemmBatch());
// Number of launch_gemm_f32 calls that ran on the SIMT kernel (process-wide).
uint64_t simt_gemm_fallbacks();

// ------------------------------------------------------------- factor (factor.cu)
constexpr int kFactorNB = 128;  // panel width of the blocked Cholesky / inverse
int64_t factor_workspace_floats(int64_t in);  // P + Dinv + T
// U may be `work` itself: U is written last, from the inverse, when the first
// in * in floats of work (P) are no longer read.  H is only read.
int run_upper_factor(const float* H, int64_t in, float damp, const int32_t* perm, float* U,
                     float* work, DeviceStatus* st, cudaStream_t stream);
int launch_act_order_perm(const double* sumsq, int64_t in, int32_t* perm, int32_t* invperm,
                          cudaStream_t stream);
int launch_identity_perm(int64_t in, int32_t* perm, int32_t* invperm, cudaStream_t stream);

// ---------------------------------------------------------------- sweep (sweep.cu)
constexpr int kSweepB = 128;
// Full blocked sweep over quantization-order weights Wq (updated in place).
// qzero != NULL: asymmetric groups, zero-points written to qzero [out, ngroups]
// (signed codes c = u - zero, What = c * scale either way).
int run_gptq_sweep(float* Wq, int64_t out, int64_t in, const float* U, int bits, int g,
                   int8_t* codes, float* qscale, uint8_t* qzero, float* Err, DeviceStatus* st,
                   cudaStream_t stream);

// ------------------------------------------------- quantize / pack / stats (quant.cu)
int launch_colstats(const uint16_t* X, int64_t n, int64_t in, double* partials, int splits,
                    double* mean_abs, double* sumsq, cudaStream_t stream);
int colstats_splits(int64_t n, int64_t in);
// Wq[r][p] = W[r][perm[p]] * cs[perm[p]]; perm and cs may be NULL.
int launch_gather_columns(const float* W, int64_t out, int64_t in, const int32_t* perm,
                          const float* cs, float* Wq, cudaStream_t stream);
// dW (bf16) and dW32 (fp32), when given, receive W0 diag(cs) - code * fp16(scale)
// (cs == NULL: W0 - code * fp16(scale)).  qzero != NULL: stored code
// u = code + zero of the (row, quantization-order group), else code + 2^(bits-1).
int launch_pack(const int8_t* codes, const float* qscale, const uint8_t* qzero,
                const int32_t* invperm, int64_t out, int64_t in, int bits, int g,
                const float* W0, const float* cs, uint32_t* qweight, uint16_t* scales16,
                uint16_t* dW, float* dW32, int32_t* g_idx, cudaStream_t stream);
// H = diag(1/s) H diag(1/s) on the upper triangle, in place; a non-finite or
// non-positive s_k sets PIQ_ERR_INVALID_ARG (where = k) in st.
int launch_scale_upper(float* H, int64_t in, const float* s, DeviceStatus* st,
                       cudaStream_t stream);
// sumsq[j] /= s_j^2 (FP64).
int launch_scale_sumsq(double* sumsq, int64_t in, const float* s, cudaStream_t stream);
int launch_awq_scale_table(const double* mean_abs, int64_t in, const float* alphas_dev,
                           int n_alpha, float* s_table, cudaStream_t stream);
int launch_awq_delta(const float* W, int64_t out, int64_t in, int bits, int g,
                     const float* s_table, int n_alpha, uint16_t* dW, cudaStream_t stream);
int launch_group_quant(const float* W, int64_t out, int64_t in, int bits, int g,
                       const float* s_table, const int* sel, int8_t* codes, float* qscale,
                       float* s_out, cudaStream_t stream);
int launch_argmin(const double* err, int n, const float* alphas_dev, int* best_idx,
                  float* best_alpha, cudaStream_t stream);
// W - What from a packed layer, into dW (bf16) or dW32 (fp32), whichever is given;
// zeros != NULL: code = u - zeros[r][grp], else u - 2^(bits-1).
int launch_dequant_delta(const float* W, int64_t out, int64_t in, const uint32_t* qweight,
                         const uint16_t* scales16, const uint8_t* zeros, const int32_t* g_idx,
                         const float* s, int bits, int g, uint16_t* dW, float* dW32,
                         DeviceStatus* st, cudaStream_t stream);

}  // namespace piq
