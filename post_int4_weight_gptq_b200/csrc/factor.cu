// Damping and the upper factor U of the inverse proxy Hessian, on the GPU.
//
// "GPTQ versus AWQ objectives", section "A strong answer" (listing): H += damp *
// mean(diag H) * I, then U = cholesky(inv(H)).T, so that inv(H_d) = U^T U.
// Section "What interviewers probe next": the damping keeps the factorization
// stable; act-order takes columns by decreasing diag(H).
//
// Route (exact identity, no explicit inverse of H): with J the index reversal,
// P = J H_d J = L L^T (lower Cholesky), then inv(H_d) = (J inv(L) J)^T (J inv(L) J)
// and J inv(L) J is upper triangular with a positive diagonal, so it is U.
//   1. lambda = damp * mean(diag H)                 (diag_mean_kernel)
//   2. P[a][b] = H[s(a)][s(b)] + lambda [a == b], s(a) = perm[in-1-a]
//   3. blocked right-looking Cholesky of P, panel width 128; each diagonal
//      block is factored and inverted in shared memory (potrf_inv_kernel), the
//      panel below is L21 = A21 inv(L11)^T and the trailing matrix is updated by
//      A22 -= L21 L21^T (FP32 SIMT GEMMs)
//   4. blocked inverse, right to left: X21 = -(X22 L21) inv(L11)
//   5. U[i][k] = X[in-1-i][in-1-k]
// A non-positive pivot sets PIQ_ERR_NOT_PD.
#include <algorithm>

#include "internal.h"

namespace piq {

namespace {

constexpr int NB = kFactorNB;      // 128
constexpr int LDS = NB + 1;        // padded shared-memory row

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

// Factor the nb x nb diagonal block at (k0, k0) of P in place (lower Cholesky)
// and write its inverse, zero-padded to nbp x nbp (nbp = 32, 64 or 128), to
// Dinv.  Rows/cols >= nb are treated as identity.
__global__ void __launch_bounds__(256) potrf_inv_kernel(float* P, int64_t ld, int64_t k0, int nb,
                                                        int nbp, float* Dinv, DeviceStatus* st) {
  extern __shared__ float sm[];
  float* S = sm;                 // [NB][LDS] factor
  float* X = sm + NB * LDS;      // [NB][LDS] inverse
  float* T = X + NB * LDS;       // [64][65] temp
  const int tid = threadIdx.x;
  if (status_bad(st)) return;

  for (int idx = tid; idx < nbp * nbp; idx += 256) {
    const int i = idx / nbp, j = idx % nbp;
    float v = 0.f;
    if (i < nb && j < nb) {
      if (j <= i) v = P[(k0 + i) * ld + (k0 + j)];
    } else if (i == j) {
      v = 1.f;
    }
    S[i * LDS + j] = v;
    X[i * LDS + j] = 0.f;
  }
  __syncthreads();

  // unblocked right-looking Cholesky
  __shared__ int bad;
  if (tid == 0) bad = 0;
  for (int j = 0; j < nbp; ++j) {
    if (tid == 0) {
      const float d = S[j * LDS + j];
      if (!(d > 0.f)) {
        bad = 1;
        set_status(st, PIQ_ERR_NOT_PD, static_cast<int>(k0 + j));
        S[j * LDS + j] = 1.f;
      } else {
        S[j * LDS + j] = sqrtf(d);
      }
    }
    __syncthreads();
    const float ljj = S[j * LDS + j];
    for (int i = j + 1 + tid; i < nbp; i += 256) S[i * LDS + j] = S[i * LDS + j] / ljj;
    __syncthreads();
    {  // trailing update of the lower triangle: one warp per row
      const int w = tid >> 5, ln = tid & 31;
      for (int i = j + 1 + w; i < nbp; i += 8) {
        const float lij = S[i * LDS + j];
        for (int k = j + 1 + ln; k <= i; k += 32)
          S[i * LDS + k] = fmaf(-lij, S[k * LDS + j], S[i * LDS + k]);
      }
    }
    __syncthreads();
  }
  if (bad) return;

  // inverse: 32 x 32 diagonal blocks by one warp each (lane = column) ...
  const int warp = tid >> 5, lane = tid & 31;
  for (int blk = warp; blk < nbp / 32; blk += 8) {
    const int o = blk * 32;
    const int c = o + lane;
    X[c * LDS + c] = 1.f / S[c * LDS + c];
    for (int i = c + 1; i < o + 32; ++i) {
      float s = 0.f;
      for (int k = c; k < i; ++k) s = fmaf(S[i * LDS + k], X[k * LDS + c], s);
      X[i * LDS + c] = -s / S[i * LDS + i];
    }
  }
  __syncthreads();
  // ... then merged pairwise: inv([[A,0],[B,C]]) has lower block -inv(C) B inv(A)
  for (int s = 32; s < nbp; s *= 2) {
    for (int pair = 0; pair < nbp / (2 * s); ++pair) {
      const int r0 = pair * 2 * s, r1 = r0 + s;
      for (int idx = tid; idx < s * s; idx += 256) {  // T = B inv(A)
        const int i = idx / s, j = idx % s;
        float acc = 0.f;
        for (int k = j; k < s; ++k) acc = fmaf(S[(r1 + i) * LDS + r0 + k], X[(r0 + k) * LDS + r0 + j], acc);
        T[i * 65 + j] = acc;
      }
      __syncthreads();
      for (int idx = tid; idx < s * s; idx += 256) {  // X21 = -inv(C) T
        const int i = idx / s, j = idx % s;
        float acc = 0.f;
        for (int k = 0; k <= i; ++k) acc = fmaf(X[(r1 + i) * LDS + r1 + k], T[k * 65 + j], acc);
        X[(r1 + i) * LDS + r0 + j] = -acc;
      }
      __syncthreads();
    }
  }

  for (int idx = tid; idx < nbp * nbp; idx += 256) {
    const int i = idx / nbp, j = idx % nbp;
    if (i < nb && j <= i) P[(k0 + i) * ld + (k0 + j)] = S[i * LDS + j];
    Dinv[idx] = (j <= i) ? X[i * LDS + j] : 0.f;
  }
}

// Copy every diagonal block's inverse into P (full nb x nb, zero above the
// diagonal) before the blocked inverse reads P as a lower-triangular X.
__global__ void put_diag_inv_kernel(float* P, int64_t in, const float* Dinv, int npanel) {
  const int pnl = blockIdx.x;
  const int64_t c0 = static_cast<int64_t>(pnl) * NB;
  const int nb = static_cast<int>(std::min<int64_t>(NB, in - c0));
  const int nbp = nb <= 32 ? 32 : (nb <= 64 ? 64 : 128);
  const float* D = Dinv + static_cast<int64_t>(pnl) * NB * NB;
  for (int idx = threadIdx.x; idx < nb * nb; idx += blockDim.x) {
    const int i = idx / nb, j = idx % nb;
    P[(c0 + i) * in + c0 + j] = D[i * nbp + j];
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

constexpr int kPotrfSmem = (2 * NB * LDS + 64 * 65) * sizeof(float);

}  // namespace

int64_t factor_workspace_floats(int64_t in) {
  const int64_t npanel = ceil_div(in, NB);
  return in * in + npanel * NB * NB + in * NB + 64;
}

int run_upper_factor(const float* H, int64_t in, float damp, const int32_t* perm, float* U,
                     float* work, DeviceStatus* st, cudaStream_t stream) {
  if (in < 1) return PIQ_ERR_INVALID_ARG;
  const int64_t npanel = ceil_div(in, NB);
  float* P = work;
  float* Dinv = P + in * in;
  float* Tb = Dinv + npanel * NB * NB;
  float* lam = Tb + in * NB;

  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPotrfSmem) != cudaSuccess)
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

  // Cholesky, panel by panel
  for (int64_t p = 0; p < npanel; ++p) {
    const int64_t k0 = p * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, in - k0));
    const int nbp = nb <= 32 ? 32 : (nb <= 64 ? 64 : 128);
    float* D = Dinv + p * NB * NB;
    note_launch();
    potrf_inv_kernel<<<1, 256, kPotrfSmem, stream>>>(P, in, k0, nb, nbp, D, st);
    if (cudaGetLastError() != cudaSuccess) return PIQ_ERR_CUDA;
    const int64_t rem = in - k0 - nb;
    if (rem <= 0) continue;
    float* A21 = P + (k0 + nb) * in + k0;
    // L21 = A21 inv(L11)^T  (in place; one CTA column since nb <= 128)
    int rc = launch_simt_gemm(static_cast<int>(rem), nb, nb, 1.f, A21, in, D, nbp, true, 0.f,
                              A21, in, 0, st, stream);
    if (rc != PIQ_OK) return rc;
    // A22 -= L21 L21^T (lower tiles)
    float* A22 = P + (k0 + nb) * in + (k0 + nb);
    rc = launch_simt_gemm(static_cast<int>(rem), static_cast<int>(rem), nb, -1.f, A21, in, A21,
                          in, true, 1.f, A22, in, 1, st, stream);
    if (rc != PIQ_OK) return rc;
  }

  // inverse of L, right to left; P becomes X = inv(L) (lower)
  note_launch();
  put_diag_inv_kernel<<<static_cast<unsigned>(npanel), 256, 0, stream>>>(P, in, Dinv,
                                                                         static_cast<int>(npanel));
  if (cudaGetLastError() != cudaSuccess) return PIQ_ERR_CUDA;
  for (int64_t p = npanel - 2; p >= 0; --p) {
    const int64_t c0 = p * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, in - c0));  // == NB here
    const int64_t c1 = c0 + nb;
    const int64_t rem = in - c1;
    const int nbp = nb <= 32 ? 32 : (nb <= 64 ? 64 : 128);
    // T = X22 L21   (X22 lower triangular, already inverted)
    int rc = launch_simt_gemm(static_cast<int>(rem), nb, static_cast<int>(rem), 1.f,
                              P + c1 * in + c1, in, P + c1 * in + c0, in, false, 0.f, Tb, NB, 2,
                              st, stream);
    if (rc != PIQ_OK) return rc;
    // X21 = -T inv(L11)
    rc = launch_simt_gemm(static_cast<int>(rem), nb, nb, -1.f, Tb, NB, Dinv + p * NB * NB, nbp,
                          false, 0.f, P + c1 * in + c0, in, 0, st, stream);
    if (rc != PIQ_OK) return rc;
  }

  {
    dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(in, 256), 64)),
              static_cast<unsigned>(std::min<int64_t>(in, 65535)));
    note_launch();
    extract_u_kernel<<<grid, 256, 0, stream>>>(P, in, U);
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
