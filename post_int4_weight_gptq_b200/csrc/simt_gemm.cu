// FP32 SIMT GEMM (FFMA) for the steps that must keep fp32 accuracy: the GPTQ
// trailing update W[:, e:] -= Err[:, b:e] U[b:e, e:] ("GPTQ versus AWQ
// objectives", remark after the listing: updates batched over column blocks
// run as GEMMs) and the panel updates of the blocked Cholesky / triangular
// inverse that produce U.
//
// 128 x 128 output tile per 256-thread CTA, 8 x 8 outputs per thread, K staged
// through double-buffered shared memory 8 at a time.  Optional batching over
// blockIdx.z with element strides, where the last entries may have fewer rows
// (and, for square triangular factors, a matching shorter K).
#include "internal.h"

namespace piq {

namespace {

constexpr int TM = 128, TN = 128, TK = 8, PAD = 4;

template <bool TRANS_B, int MODE>
__global__ void __launch_bounds__(256)
    simt_gemm_kernel(int M, int N, int K, float alpha, const float* A, int64_t lda,
                     const float* B, int64_t ldb, float beta, float* C, int64_t ldc,
                     GemmBatch bt, const DeviceStatus* st) {
  const int m0 = blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;
  if (MODE == 1 && n0 >= m0 + TM) return;  // tile strictly above the diagonal
  if (status_bad(st)) return;
  const int z = blockIdx.z;
  if (bt.count > 1) {
    A += z * bt.stride_a;
    B += z * bt.stride_b;
    C += z * bt.stride_c;
  }
  if (bt.m_total > 0) {  // ragged last entries
    const int64_t mz = bt.m_total - static_cast<int64_t>(z) * bt.m_step;
    if (mz < M) M = static_cast<int>(mz);
    if (bt.k_follows_m) K = M;
    if (M <= 0 || m0 >= M) return;
  }
  // K range that can be nonzero: mode 2, A lower (k <= row); mode 3, op(B)
  // upper (k <= col); mode 4, op(B) lower (k >= col)
  const int kend = (MODE == 2) ? min(K, m0 + TM) : (MODE == 3) ? min(K, n0 + TN) : K;
  const int kbeg = (MODE == 4) ? min(K, n0) & ~(TK - 1) : 0;

  __shared__ __align__(16) float As[2][TK][TM + PAD];
  __shared__ __align__(16) float Bs[2][TK][TN + PAD];

  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;

  // global -> register staging indices
  const int a_r = tid >> 1, a_k = (tid & 1) * 4;
  const int b_k = TRANS_B ? (tid & 1) * 4 : (tid >> 5);
  const int b_n = TRANS_B ? (tid >> 1) : (tid & 31) * 4;

  float ra[4], rb[4];
  auto load_tiles = [&](int k0) {
    const int gr = m0 + a_r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int gk = k0 + a_k + i;
      ra[i] = (gr < M && gk < kend) ? A[static_cast<int64_t>(gr) * lda + gk] : 0.f;
    }
    if (TRANS_B) {
      const int gn = n0 + b_n;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int gk = k0 + b_k + i;
        rb[i] = (gn < N && gk < kend) ? B[static_cast<int64_t>(gn) * ldb + gk] : 0.f;
      }
    } else {
      const int gk = k0 + b_k;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int gn = n0 + b_n + i;
        rb[i] = (gn < N && gk < kend) ? B[static_cast<int64_t>(gk) * ldb + gn] : 0.f;
      }
    }
  };
  auto store_tiles = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 4; ++i) As[buf][a_k + i][a_r] = ra[i];
    if (TRANS_B) {
#pragma unroll
      for (int i = 0; i < 4; ++i) Bs[buf][b_k + i][b_n] = rb[i];
    } else {
      *reinterpret_cast<float4*>(&Bs[buf][b_k][b_n]) = make_float4(rb[0], rb[1], rb[2], rb[3]);
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  int buf = 0;
  if (kend > kbeg) {
    load_tiles(kbeg);
    store_tiles(0);
  }
  __syncthreads();
  for (int k0 = kbeg; k0 < kend; k0 += TK) {
    const bool more = k0 + TK < kend;
    if (more) load_tiles(k0 + TK);
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[8], b[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      store_tiles(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (c >= N) continue;
      float* dst = C + static_cast<int64_t>(r) * ldc + c;
      const float v = alpha * acc[i][j];
      *dst = (beta != 0.f) ? fmaf(beta, *dst, v) : v;
    }
  }
}

template <bool TB, int MODE>
int launch_one(int M, int N, int K, float alpha, const float* A, int64_t lda, const float* B,
               int64_t ldb, float beta, float* C, int64_t ldc, const GemmBatch& bt,
               const DeviceStatus* st, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(ceil_div(N, TN)), static_cast<unsigned>(ceil_div(M, TM)),
            static_cast<unsigned>(bt.count));
  note_launch();
  simt_gemm_kernel<TB, MODE><<<grid, 256, 0, stream>>>(M, N, K, alpha, A, lda, B, ldb, beta, C,
                                                       ldc, bt, st);
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace

int launch_simt_gemm(int M, int N, int K, float alpha, const float* A, int64_t lda,
                     const float* B, int64_t ldb, bool trans_b, float beta, float* C,
                     int64_t ldc, int mode, const DeviceStatus* st, cudaStream_t stream,
                     const GemmBatch& bt) {
  if (M <= 0 || N <= 0 || bt.count < 1) return PIQ_OK;
  if (ceil_div(M, TM) > 65535 || bt.count > 65535) return PIQ_ERR_INVALID_ARG;
#define PIQ_GEMM_CASE(TB, MD)                                                              \
  if (trans_b == TB && mode == MD)                                                         \
    return launch_one<TB, MD>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, bt, st, stream);
  PIQ_GEMM_CASE(true, 0)
  PIQ_GEMM_CASE(true, 1)
  PIQ_GEMM_CASE(true, 3)
  PIQ_GEMM_CASE(false, 0)
  PIQ_GEMM_CASE(false, 2)
  PIQ_GEMM_CASE(false, 3)
  PIQ_GEMM_CASE(false, 4)
#undef PIQ_GEMM_CASE
  return PIQ_ERR_INVALID_ARG;
}

}  // namespace piq
