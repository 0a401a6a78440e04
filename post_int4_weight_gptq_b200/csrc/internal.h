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
// H = X^T X with FP64 sums (128-sample tensor-core chunks added in FP64):
// upper triangle of a [in, in] fp64 matrix (syrk64.cu).
int launch_syrk64(const uint16_t* X, int64_t n, int64_t in, double* H, DeviceStatus* st,
                  cudaStream_t stream);
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
int run_error_via_h(const float* D, int64_t out, int64_t in, const double* H, uint16_t* dsplit,
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

// ------------------------------------ FP64-grade GEMM on the INT8 tensor cores (ozaki.cu)
// A matrix as s signed 7-bit digits per entry, scaled per row by 2^ex[row]:
// q[i][row][kpad] int8 (K-major, zero padded to kpad), ex[row] int32.
constexpr int kMaxDigits = 7;
constexpr int kFactorDigits = 5;  // Cholesky panel products: ~1e-10 relative
constexpr int kSweepDigits = 5;   // GPTQ block updates: ~1e-10 relative
struct DigitMat {
  int8_t* q = nullptr;
  int* ex = nullptr;
  int64_t rows = 0, kpad = 0;
  int s = 0;
  int64_t plane = 0;  // bytes between digit planes (0: rows * kpad, a matrix of its own)
  // rows [r0, r0 + n) of this matrix, the planes of the whole one
  DigitMat rows_from(int64_t r0, int64_t n) const {
    DigitMat v = *this;
    v.q = q + r0 * kpad;
    v.ex = ex + r0;
    v.rows = n;
    v.plane = plane ? plane : rows * kpad;
    return v;
  }
};
// Per-launch timing of the digit GEMM while phase timing is on: begin
// records an event before the launch and returns a slot (-1 when off), end
// records one after it with the launch's algorithmic INT8 operations.
int gemm_timing_begin(cudaStream_t stream);
void gemm_timing_end(int slot, cudaStream_t stream, double int8_ops);
int64_t digit_kpad(int64_t K);  // K rounded up to a multiple of 64
// Digits of the rows x K matrix whose entry (r, k) is src[r * rs + k * ks]
// (strides may be negative); out->rows, kpad and s must match.
int launch_slice(const double* src, int64_t rs, int64_t ks, int64_t rows, int64_t K, int s,
                 DigitMat* out, cudaStream_t stream);
// C[r][c] (+)= alpha sum_k A(r, k) B(c, k) for r < M, c < N, C fp64 row-major;
// beta 0 stores, 1 adds; lower != 0 touches only c <= r.
int launch_ozaki_gemm(int64_t M, int64_t N, const DigitMat& A, const DigitMat& B, double alpha,
                      int beta, int lower, double* C, int64_t ldc, DeviceStatus* st,
                      cudaStream_t stream, int max_ctas = 0);

// ---------------------------------------------- FP64-grade factor (factor64.cu)
// L = chol(J H_p J + lambda I) in fp64 (lower, row-major [in][in] inside
// `work`); R = J L J is the upper factor with H_d = R R^T and U = inv(R).
int64_t factor64_workspace_bytes(int64_t in);
int run_factor64(const double* H, int64_t in, float damp, const int32_t* perm, void* work,
                 double** L_out, DeviceStatus* st, cudaStream_t stream);
// Ub[blk] = inv(R[b:e, b:e]) (128 x 128 fp64) for the blocks [starts[blk], starts[blk+1]).
int launch_block_inverses(const double* L, int64_t in, const int64_t* starts_dev, int nblocks,
                          double* Ub, cudaStream_t stream);

// ------------------------------------------------ FP64 sweep on R (sweep64.cu)
struct Sweep64Ws {
  int nblocks = 0;
  double* acc = nullptr;     // [out][in] accumulated updates
  double* Ub = nullptr;      // [nblocks][128][128]
  int64_t* starts = nullptr; // [nblocks + 1]
  int8_t* dq = nullptr;      // digits of W0 - Q of one block [s][out][128]
  int* dex = nullptr;
  int8_t* rq = nullptr;      // digits of one block row of R [s][in][128]
  int* rex = nullptr;
  double* yscr = nullptr;    // group scales wider than a block
  double* dsb = nullptr;     // W0 - Q of a superblock [out][1024] (fp64)
  int8_t* sbq = nullptr;     // its digits, and those of R's rows of the superblock
  int* sbex = nullptr;
  int8_t* sbrq = nullptr;
  int* sbrex = nullptr;
};
int sweep64_blocks(int64_t in, int g);
int64_t carve_sweep64(void* base, int64_t out, int64_t in, int g, Sweep64Ws* w);
int64_t sweep64_workspace_bytes(int64_t out, int64_t in, int g);
// Codes and scales (and zero-points) of the listing's loop over W0 (quantization
// order, fp32, not modified) with the factor L of run_factor64.
int run_gptq_sweep64(const float* W0, int64_t out, int64_t in, const double* L, int bits, int g,
                     int8_t* codes, float* qscale, uint8_t* qzero, const Sweep64Ws& w,
                     DeviceStatus* st, cudaStream_t stream);

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
int launch_scale_upper(double* H, int64_t in, const float* s, DeviceStatus* st,
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
