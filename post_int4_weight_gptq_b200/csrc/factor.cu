// Damping and the upper factor U of the inverse proxy Hessian, on the GPU.
//
// "GPTQ versus AWQ objectives", section "A strong answer" (listing): H += damp *
// mean(diag H) * I, then U = cholesky(inv(H)).T, so that inv(H_d) = U^T U.
// Section "What interviewers probe next": the damping keeps the factorization
// stable; act-order takes columns by decreasing diag(H).
//
// Route (exact identity, no inverse of H): with J the index reversal,
// P = J H_d J = L L^T (lower Cholesky), then inv(H_d) = (J inv(L) J)^T (J inv(L) J)
// and J inv(L) J is upper triangular with a positive diagonal, so it is U.
//   1. lambda = damp * mean(diag H)                        (diag_mean_kernel)
//   2. P[a][b] = H[s(a)][s(b)] + lambda [a == b], s(a) = perm[in-1-a]
//   3. right-looking blocked Cholesky, 128-wide panels: each diagonal block is
//      factored and inverted in shared memory (chol_inv_kernel), the panel
//      below is L21 = A21 inv(L11)^T and the trailing matrix A22 -= L21 L21^T
//      (FP32 SIMT GEMMs that skip the zero triangles)
//   4. X = inv(L) from the diagonal inverses, merging pairs of s-blocks level by
//      level (s = 128, 256, ...): X21 = -X22 (L21 X11), every pair of a level in
//      one batched launch
//   5. U[i][k] = X[in-1-i][in-1-k]
// A non-positive pivot sets PIQ_ERR_NOT_PD.
#include <algorithm>

#include "internal.h"

namespace piq {

namespace {

constexpr int NB = kFactorNB;  // 128
constexpr int LDS = NB + 1;    // padded shared-memory row

__global__ void diag_mean_kernel(const float* H, int64_t in, float damp, DeviceStatus* st,
                                 float* lambda_f) {
  __shared__ double sh[256];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < in; i += 256) acc += static_cast<double>(H[i * in + i]);
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double lam = static_cast<double>(damp) * (sh[0] / static_cast<double>(in));
    st->lambda = lam;
    *lambda_f = static_cast<float>(lam);
  }
}

// P (lower part, b <= a) from the upper triangle of H.  32 x 32 tiles.
__global__ void build_rev_kernel(const float* H, int64_t in, const int32_t* perm,
                                 const float* lambda_f, float* P) {
  const int64_t a0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * 32;
  if (b0 > a0 + 31) return;
  const float lam = *lambda_f;
  const int64_t b = b0 + threadIdx.x;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int64_t a = a0 + r;
    if (a >= in || b >= in || b > a) continue;
    const int64_t x = perm ? perm[in - 1 - a] : in - 1 - a;
    const int64_t y = perm ? perm[in - 1 - b] : in - 1 - b;
    const int64_t lo = x < y ? x : y, hi = x < y ? y : x;
    float v = H[lo * in + hi];
    if (a == b) v += lam;
    P[a * in + b] = v;
  }
}

constexpr int SP = 16;  // sub-panel width inside a 128 block
constexpr unsigned FULL = 0xffffffffu;

// One warp factors a 16 x 16 SPD block and inverts its factor, in registers.
// Lane i < 16 holds row i: on entry a[k] = A[i][k] (k <= i); on exit a[k] =
// L[i][k] and x[k] = inv(L)[i][k] (0 above the diagonal).  Lanes >= 16 carry
// zeros.  Template recursion keeps register indices compile-time; the code is
// small enough for the instruction cache.
template <int J>
__device__ __forceinline__ void chol16_col(float (&a)[SP], float& rdiag, int lane, bool& ok) {
  if constexpr (J < SP) {
    const float d = __shfl_sync(FULL, a[J], J);
    ok = ok && (d > 0.f);
    const float dd = d > 0.f ? d : 1.f;
    const float r = rsqrtf(dd);  // 1 / L_JJ
    const float ljj = dd * r;     // L_JJ
    if (lane == J) rdiag = r;
    const float lij = (lane > J) ? a[J] * r : (lane == J ? ljj : 0.f);
    a[J] = lij;
#pragma unroll
    for (int k = J + 1; k < SP; ++k) {
      const float lkj = __shfl_sync(FULL, lij, k);
      if (k <= lane) a[k] = fmaf(-lij, lkj, a[k]);
    }
    chol16_col<J + 1>(a, rdiag, lane, ok);
  }
}

// forward substitution by rows: X_K = (e_K - sum_{c<K} L_Kc X_c) / L_KK
template <int K>
__device__ __forceinline__ void inv16_row(const float (&a)[SP], float (&x)[SP], float rdiag,
                                          int lane) {
  if constexpr (K < SP) {
    if (lane == K) {
#pragma unroll
      for (int c = 0; c <= K; ++c) x[c] *= rdiag;
    }
#pragma unroll
    for (int c = 0; c <= K; ++c) {
      const float xkc = __shfl_sync(FULL, x[c], K);
      if (lane > K) x[c] = fmaf(-a[K], xkc, x[c]);
    }
    inv16_row<K + 1>(a, x, rdiag, lane);
  }
}

// z[c] = sum_{k <= c} y[k] * Xd[c][k]   (row times the transposed lower inverse)
template <int C>
__device__ __forceinline__ void trsm_col(const float (&y)[SP], float (&z)[SP], const float* Xd) {
  if constexpr (C < SP) {
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k <= C; ++k) acc = fmaf(y[k], Xd[C * LDS + k], acc);
    z[C] = acc;
    trsm_col<C + 1>(y, z, Xd);
  }
}

// Factor the nb x nb diagonal block of P at (o, o) in place (lower Cholesky) and
// write its inverse to X at (o, o) (full nb x nb, zeros above the diagonal).
// Rows/cols >= nb are padded with the identity up to nbp = 32, 64 or 128.
constexpr int CI_THREADS = 512;
constexpr int CI_WARPS = CI_THREADS / 32;

__global__ void __launch_bounds__(CI_THREADS)
    chol_inv_kernel(float* P, float* X, int64_t ld, int64_t o, int nb, int nbp,
                    DeviceStatus* st) {
  extern __shared__ float sm[];
  float* S = sm;              // [NB][LDS] factor
  float* Xs = sm + NB * LDS;  // [NB][LDS] inverse
  float* T = Xs + NB * LDS;   // [64][65] temp
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (status_bad(st)) return;
  if (tid == 0) bad = 0;

  for (int i = warp; i < nbp; i += CI_WARPS) {
    for (int j = lane; j < nbp; j += 32) {
      if (i < nb && j <= i)
        cp_async4(S + i * LDS + j, P + (o + i) * ld + (o + j));
      else
        S[i * LDS + j] = (i == j) ? 1.f : 0.f;
      Xs[i * LDS + j] = 0.f;
    }
  }
  cp_async_wait_all();
  __syncthreads();

  // right-looking over 16-wide sub-panels
  for (int c0 = 0; c0 < nbp; c0 += SP) {
    if (warp == 0) {
      float a[SP], x[SP];
      float rdiag = 0.f;
      bool ok = true;
#pragma unroll
      for (int k = 0; k < SP; ++k) a[k] = (lane < SP) ? S[(c0 + lane) * LDS + c0 + k] : 0.f;
      chol16_col<0>(a, rdiag, lane, ok);
#pragma unroll
      for (int k = 0; k < SP; ++k) {
        a[k] = (k <= lane) ? a[k] : 0.f;
        x[k] = (k == lane) ? 1.f : 0.f;
      }
      inv16_row<0>(a, x, rdiag, lane);
      if (!ok && lane == 0) {
        bad = 1;
        set_status(st, PIQ_ERR_NOT_PD, static_cast<int>(o + c0));
      }
      if (lane < SP) {
#pragma unroll
        for (int k = 0; k < SP; ++k) {
          S[(c0 + lane) * LDS + c0 + k] = a[k];
          Xs[(c0 + lane) * LDS + c0 + k] = x[k];
        }
      }
    }
    __syncthreads();
    if (bad) return;
    const int r0 = c0 + SP;
    if (r0 < nbp) {
      // L21 = A21 inv(L11)^T, one thread per row
      const int r = r0 + tid;
      if (r < nbp) {
        float y[SP], z[SP];
#pragma unroll
        for (int k = 0; k < SP; ++k) y[k] = S[r * LDS + c0 + k];
        trsm_col<0>(y, z, Xs + c0 * LDS + c0);
#pragma unroll
        for (int cc = 0; cc < SP; ++cc) S[r * LDS + c0 + cc] = z[cc];
      }
      __syncthreads();
      // A22 -= L21 L21^T (lower triangle), one warp per row
      for (int i = r0 + warp; i < nbp; i += CI_WARPS) {
        for (int j = r0 + lane; j <= i; j += 32) {
          float acc = S[i * LDS + j];
#pragma unroll
          for (int k = 0; k < SP; ++k)
            acc = fmaf(-S[i * LDS + c0 + k], S[j * LDS + c0 + k], acc);
          S[i * LDS + j] = acc;
        }
      }
      __syncthreads();
    }
  }

  // inverse of the whole block from the diagonal 16-blocks:
  // inv([[A,0],[B,C]]) has lower-left block -inv(C) B inv(A)
  for (int s = SP; s < nbp; s *= 2) {
    for (int pr = 0; pr < nbp / (2 * s); ++pr) {
      const int q0 = pr * 2 * s, q1 = q0 + s;
      for (int i = warp; i < s; i += CI_WARPS) {  // T = B inv(A)
        for (int j = lane; j < s; j += 32) {
          float acc = 0.f;
          for (int k = j; k < s; ++k)
            acc = fmaf(S[(q1 + i) * LDS + q0 + k], Xs[(q0 + k) * LDS + q0 + j], acc);
          T[i * 65 + j] = acc;
        }
      }
      __syncthreads();
      for (int i = warp; i < s; i += CI_WARPS) {  // X21 = -inv(C) T
        for (int j = lane; j < s; j += 32) {
          float acc = 0.f;
          for (int k = 0; k <= i; ++k) acc = fmaf(Xs[(q1 + i) * LDS + q1 + k], T[k * 65 + j], acc);
          Xs[(q1 + i) * LDS + q0 + j] = -acc;
        }
      }
      __syncthreads();
    }
  }

  for (int i = warp; i < nb; i += CI_WARPS) {
    for (int j = lane; j < nb; j += 32) {
      if (j <= i) P[(o + i) * ld + (o + j)] = S[i * LDS + j];
      X[(o + i) * ld + (o + j)] = (j <= i) ? Xs[i * LDS + j] : 0.f;
    }
  }
}

// U[i][k] = X[in-1-i][in-1-k] for k >= i, else 0.
__global__ void extract_u_kernel(const float* X, int64_t in, float* U) {
  for (int64_t i = blockIdx.y; i < in; i += gridDim.y) {
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < in;
         k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      U[i * in + k] = (k >= i) ? X[(in - 1 - i) * in + (in - 1 - k)] : 0.f;
    }
  }
}

// rank of each column by decreasing sumsq (exact FP64 column sums of squares,
// i.e. diag(X^T X)); equal values keep index order.
__global__ void act_order_rank_kernel(const double* d, int64_t in, int32_t* perm,
                                      int32_t* invperm) {
  __shared__ double tile[1024];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const double di = i < in ? d[i] : 0.0;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < in; j0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x)
      tile[t] = (j0 + t < in) ? d[j0 + t] : 0.0;
    __syncthreads();
    const int lim = static_cast<int>(std::min<int64_t>(1024, in - j0));
    if (i < in) {
      for (int t = 0; t < lim; ++t) {
        const double dj = tile[t];
        const int64_t j = j0 + t;
        rank += (dj > di) || (dj == di && j < i);
      }
    }
  }
  if (i < in) {
    perm[rank] = static_cast<int32_t>(i);
    invperm[i] = static_cast<int32_t>(rank);
  }
}

__global__ void identity_perm_kernel(int64_t in, int32_t* perm, int32_t* invperm) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < in) {
    if (perm) perm[i] = static_cast<int32_t>(i);
    if (invperm) invperm[i] = static_cast<int32_t>(i);
  }
}

constexpr int kCholSmem = (2 * NB * LDS + 64 * 65) * sizeof(float);

// Floats of the pair scratch of the level-by-level inverse: max over levels of
// (pairs at that level) * s * s.
int64_t trtri_scratch_floats(int64_t n) {
  int64_t best = 0;
  for (int64_t s = NB; s < n; s *= 2) {
    const int64_t pairs = ceil_div(n - s, 2 * s);
    best = std::max(best, pairs * s * s);
  }
  return best;
}

}  // namespace

int64_t factor_workspace_floats(int64_t in) {
  return 2 * in * in + trtri_scratch_floats(in) + 64;  // P, X, pair scratch, lambda
}

int run_upper_factor(const float* H, int64_t in, float damp, const int32_t* perm, float* U,
                     float* work, DeviceStatus* st, cudaStream_t stream) {
  if (in < 1) return PIQ_ERR_INVALID_ARG;
  float* P = work;
  float* X = P + in * in;
  float* T = X + in * in;
  float* lam = T + trtri_scratch_floats(in);
  const int64_t ld = in;

  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kCholSmem) != cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }

  note_launch();
  diag_mean_kernel<<<1, 256, 0, stream>>>(H, in, damp, st, lam);
  {
    dim3 grid(static_cast<unsigned>(ceil_div(in, 32)), static_cast<unsigned>(ceil_div(in, 32)));
    note_launch();
    build_rev_kernel<<<grid, dim3(32, 8), 0, stream>>>(H, in, perm, lam, P);
  }
  if (cudaGetLastError() != cudaSuccess) return PIQ_ERR_CUDA;

  // 3. Cholesky, panel by panel; diagonal inverses land in X
  for (int64_t k0 = 0; k0 < in; k0 += NB) {
    const int nb = static_cast<int>(std::min<int64_t>(NB, in - k0));
    const int nbp = nb <= 32 ? 32 : (nb <= 64 ? 64 : 128);
    note_launch();
    chol_inv_kernel<<<1, CI_THREADS, kCholSmem, stream>>>(P, X, ld, k0, nb, nbp, st);
    if (cudaGetLastError() != cudaSuccess) return PIQ_ERR_CUDA;
    const int rem = static_cast<int>(in - k0 - nb);
    if (rem <= 0) continue;
    float* A21 = P + (k0 + nb) * ld + k0;
    const float* X11 = X + k0 * ld + k0;
    // L21 = A21 X11^T in place (nb <= 128: one CTA column)
    int rc = launch_gemm_f32(rem, nb, nb, 1.f, A21, ld, X11, ld, true, 0.f, A21, ld, 3, st,
                              stream);
    if (rc != PIQ_OK) return rc;
    // A22 -= L21 L21^T (lower tiles)
    rc = launch_gemm_f32(rem, rem, nb, -1.f, A21, ld, A21, ld, true, 1.f,
                          P + (k0 + nb) * ld + (k0 + nb), ld, 1, st, stream);
    if (rc != PIQ_OK) return rc;
  }

  // 4. X = inv(L): merge pairs of s-blocks, all pairs of a level per launch
  for (int64_t s = NB; s < in; s *= 2) {
    const int64_t pairs = ceil_div(in - s, 2 * s);
    GemmBatch bt;
    bt.count = static_cast<int>(pairs);
    bt.m_total = in - s;
    bt.m_step = 2 * s;
    const int si = static_cast<int>(s);
    // T_p = L21_p X11_p   (X11 lower, used as is)
    bt.stride_a = 2 * s * (ld + 1);
    bt.stride_b = 2 * s * (ld + 1);
    bt.stride_c = s * s;
    int rc = launch_gemm_f32(si, si, si, 1.f, P + s * ld, ld, X, ld, false, 0.f, T, s, 4, st,
                              stream, bt);
    if (rc != PIQ_OK) return rc;
    // X21_p = -X22_p T_p   (X22 lower, K = its rows)
    bt.stride_a = 2 * s * (ld + 1);
    bt.stride_b = s * s;
    bt.stride_c = 2 * s * (ld + 1);
    bt.k_follows_m = true;
    rc = launch_gemm_f32(si, si, si, -1.f, X + s * ld + s, ld, T, s, false, 0.f, X + s * ld, ld,
                          2, st, stream, bt);
    if (rc != PIQ_OK) return rc;
  }

  {
    dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(in, 256), 64)),
              static_cast<unsigned>(std::min<int64_t>(in, 65535)));
    note_launch();
    extract_u_kernel<<<grid, 256, 0, stream>>>(X, in, U);
  }
  return cudaGetLastError() == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

int launch_act_order_perm(const double* sumsq, int64_t in, int32_t* perm, int32_t* invperm,
                          cudaStream_t stream) {
  note_launch();
  act_order_rank_kernel<<<static_cast<unsigned>(ceil_div(in, 256)), 256, 0, stream>>>(
      sumsq, in, perm, invperm);
  return cudaGetLastError() == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

int launch_identity_perm(int64_t in, int32_t* perm, int32_t* invperm, cudaStream_t stream) {
  note_launch();
  identity_perm_kernel<<<static_cast<unsigned>(ceil_div(in, 256)), 256, 0, stream>>>(in, perm,
                                                                                     invperm);
  return cudaGetLastError() == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace piq
