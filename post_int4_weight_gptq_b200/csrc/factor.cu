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
//      (FP32-accurate tensor-core GEMMs, three TF32 passes, that skip the zero
//      triangles)
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
constexpr int SLD = NB + 4;    // shared-memory row stride (float4-aligned rows)

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

// One warp factors a 16 x 16 SPD block, in registers.  Lane i < 16 holds row
// i: on entry a[k] = A[i][k] (k <= i); on exit a[k] = L[i][k] (k <= i) and
// rdiag = 1 / L_ii.  Lanes >= 16 carry zeros.  d is pivot J, already
// broadcast.  The next pivot is formed by lane J+1 from its own values and
// shuffled first (the serial chain per pivot: one shuffle, one rsqrt, a
// multiply and an FMA); the rest of column J reaches the lanes through shared
// memory (one store, four broadcast float4 loads, double-buffered by pivot
// parity) instead of fifteen shuffles.  Template recursion keeps register
// indices compile-time.
template <int J>
__device__ __forceinline__ void chol16_col(float (&a)[SP], float& rdiag, int lane, bool& ok,
                                           float d, float* colbuf) {
  if constexpr (J < SP) {
    ok = ok && (d > 0.f);
    const float dd = d > 0.f ? d : 1.f;
    const float r = rsqrtf(dd);  // 1 / L_JJ
    const float ljj = dd * r;     // L_JJ
    if (lane == J) rdiag = r;
    const float lij = (lane > J) ? a[J] * r : (lane == J ? ljj : 0.f);
    a[J] = lij;
    float dn = 0.f;
    if constexpr (J + 1 < SP) {
      dn = __shfl_sync(FULL, fmaf(-lij, lij, a[J + 1]), J + 1);
      float* col = colbuf + (J & 1) * SP;
      if (lane < SP) col[lane] = lij;
      __syncwarp();
      float lk[SP];
#pragma unroll
      for (int q = (J + 1) / 4; q < SP / 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(col)[q];
        lk[4 * q] = v.x;
        lk[4 * q + 1] = v.y;
        lk[4 * q + 2] = v.z;
        lk[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int k = J + 1; k < SP; ++k)
        if (k <= lane) a[k] = fmaf(-lij, lk[k], a[k]);
    }
    chol16_col<J + 1>(a, rdiag, lane, ok, dn, colbuf);
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

// Forward substitution of one row against the 16 x 16 factor L11 (rows of
// Ld, stride SLD) with the reciprocal pivots rv: on entry y = a row of A21, on
// exit y = that row of A21 inv(L11)^T.
template <int C>
__device__ __forceinline__ void trsm_sub(float (&y)[SP], const float* Ld, const float* rv) {
  if constexpr (C < SP) {
    y[C] *= rv[C];
#pragma unroll
    for (int c = C + 1; c < SP; ++c) y[c] = fmaf(-y[C], Ld[c * SLD + C], y[c]);
    trsm_sub<C + 1>(y, Ld, rv);
  }
}

__device__ __forceinline__ void fma4x4(float (&acc)[4][4], const float4 a, const float4 b) {
  const float av[4] = {a.x, a.y, a.z, a.w};
  const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
}

// Triangular index t -> (row tile bi, col tile bj), bj <= bi.
__device__ __forceinline__ void tri_index(int t, int& bi, int& bj) {
  int r = static_cast<int>((sqrtf(8.f * static_cast<float>(t) + 1.f) - 1.f) * 0.5f);
  while ((r + 1) * (r + 2) / 2 <= t) ++r;
  while (r * (r + 1) / 2 > t) --r;
  bi = r;
  bj = t - r * (r + 1) / 2;
}

// Factor the nb x nb diagonal block of P at (o, o) in place (lower Cholesky) and
// write its inverse to X at (o, o) (full nb x nb, zeros above the diagonal).
// Rows/cols >= nb are padded with the identity up to nbp = 32, 64 or 128.
//
// Right-looking over 16-wide sub-panels: warp 0 factors the 16 x 16 diagonal
// block in registers (the only serial part: one pivot after the other); the
// rows below are solved against it by substitution, one thread per row, and
// the trailing lower triangle is updated in 4 x 4 register tiles from a
// transposed copy of the panel (float4 loads).  The inverse is formed at the
// end: the 16 x 16 diagonal inverses in parallel (one warp each), then pairs of
// s-blocks merged level by level, inv([[A,0],[B,C]]) having lower-left block
// -inv(C) B inv(A), again in 4 x 4 register tiles.
constexpr int CI_THREADS = 512;
constexpr int CI_WARPS = CI_THREADS / 32;
constexpr int TLD = 64 + 4;  // merge temp row stride

__global__ void __launch_bounds__(CI_THREADS)
    chol_inv_kernel(float* P, float* X, int64_t ld, int64_t o, int nb, int nbp,
                    DeviceStatus* st) {
  extern __shared__ __align__(16) float sm[];
  float* S = sm;                 // [NB][SLD] factor
  float* Xs = S + NB * SLD;      // [NB][SLD] inverse
  float* LT = Xs + NB * SLD;     // [SP][SLD] current panel, transposed
  float* Tm = LT + SP * SLD;     // [64][TLD] merge temp
  float* rinv = Tm + 64 * TLD;   // [NB] reciprocal pivots
  float* colbuf = rinv + NB;     // [2][SP] pivot-column broadcast (16-byte aligned)
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  pdl_wait();  // P comes from the previous kernel
  if (status_bad(st)) return;
  if (tid == 0) bad = 0;

  for (int i = warp; i < nbp; i += CI_WARPS) {
    for (int j = lane; j < nbp; j += 32) {
      if (i < nb && j <= i)
        cp_async4(S + i * SLD + j, P + (o + i) * ld + (o + j));
      else
        S[i * SLD + j] = (i == j) ? 1.f : 0.f;
      Xs[i * SLD + j] = 0.f;
    }
  }
  cp_async_wait_all();
  __syncthreads();

  for (int c0 = 0; c0 < nbp; c0 += SP) {
    // ---- the 16 x 16 diagonal block (warp 0)
    if (warp == 0) {
      float a[SP];
      float rdiag = 0.f;
      bool ok = true;
      if (lane < SP) {
        const float4* row = reinterpret_cast<const float4*>(S + (c0 + lane) * SLD + c0);
#pragma unroll
        for (int q = 0; q < SP / 4; ++q) {
          const float4 v = row[q];
          a[4 * q] = v.x;
          a[4 * q + 1] = v.y;
          a[4 * q + 2] = v.z;
          a[4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < SP; ++k) a[k] = 0.f;
      }
      chol16_col<0>(a, rdiag, lane, ok, __shfl_sync(FULL, a[0], 0), colbuf);
      if (!ok && lane == 0) {
        bad = 1;
        set_status(st, PIQ_ERR_NOT_PD, static_cast<int>(o + c0));
      }
      if (lane < SP) {
        float4* row = reinterpret_cast<float4*>(S + (c0 + lane) * SLD + c0);
#pragma unroll
        for (int q = 0; q < SP / 4; ++q)
          row[q] = make_float4(4 * q <= lane ? a[4 * q] : 0.f, 4 * q + 1 <= lane ? a[4 * q + 1] : 0.f,
                               4 * q + 2 <= lane ? a[4 * q + 2] : 0.f,
                               4 * q + 3 <= lane ? a[4 * q + 3] : 0.f);
        rinv[c0 + lane] = rdiag;
      }
    }
    __syncthreads();
    if (bad) return;
    const int r0 = c0 + SP;
    if (r0 >= nbp) break;
    // ---- L21 = A21 inv(L11)^T, one thread per row; also the transposed copy
    {
      const int r = r0 + tid;
      if (r < nbp) {
        float y[SP];
        float4* row = reinterpret_cast<float4*>(S + r * SLD + c0);
#pragma unroll
        for (int q = 0; q < SP / 4; ++q) {
          const float4 v = row[q];
          y[4 * q] = v.x;
          y[4 * q + 1] = v.y;
          y[4 * q + 2] = v.z;
          y[4 * q + 3] = v.w;
        }
        trsm_sub<0>(y, S + c0 * SLD + c0, rinv + c0);
#pragma unroll
        for (int q = 0; q < SP / 4; ++q)
          row[q] = make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]);
#pragma unroll
        for (int k = 0; k < SP; ++k) LT[k * SLD + r] = y[k];
      }
    }
    __syncthreads();
    // ---- A22 -= L21 L21^T on the lower 4 x 4 tiles
    {
      const int mt = (nbp - r0) / 4;
      const int ntile = mt * (mt + 1) / 2;
      for (int t = tid; t < ntile; t += CI_THREADS) {
        int bi, bj;
        tri_index(t, bi, bj);
        const int i0 = r0 + 4 * bi, j0 = r0 + 4 * bj;
        float acc[4][4] = {};
#pragma unroll
        for (int k = 0; k < SP; ++k)
          fma4x4(acc, *reinterpret_cast<const float4*>(LT + k * SLD + i0),
                 *reinterpret_cast<const float4*>(LT + k * SLD + j0));
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float4* dst = reinterpret_cast<float4*>(S + (i0 + x) * SLD + j0);
          float4 v = *dst;
          v.x -= acc[x][0];
          v.y -= acc[x][1];
          v.z -= acc[x][2];
          v.w -= acc[x][3];
          *dst = v;
        }
      }
    }
    __syncthreads();
  }

  // ---- diagonal 16 x 16 inverses, one warp each
  for (int w = warp; w < nbp / SP; w += CI_WARPS) {
    const int c0 = w * SP;
    float a[SP], x[SP];
    const float rdiag = lane < SP ? rinv[c0 + lane] : 0.f;
#pragma unroll
    for (int k = 0; k < SP; ++k) {
      a[k] = (lane < SP && k <= lane) ? S[(c0 + lane) * SLD + c0 + k] : 0.f;
      x[k] = (k == lane) ? 1.f : 0.f;
    }
    inv16_row<0>(a, x, rdiag, lane);
    if (lane < SP) {
#pragma unroll
      for (int k = 0; k < SP; ++k) Xs[(c0 + lane) * SLD + c0 + k] = x[k];
    }
  }
  __syncthreads();

  // ---- merges: for each pair (q0, q1 = q0 + s) at level s,
  //      T = L[q1.., q0..] inv(L)[q0.., q0..]   then   X21 = -inv(L)[q1.., q1..] T
  for (int s = SP; s < nbp; s *= 2) {
    const int per = (s / 4) * (s / 4);   // 4 x 4 tiles per pair
    const int npair = nbp / (2 * s);
    for (int t = tid; t < per * npair; t += CI_THREADS) {
      const int pr = t / per, u = t - pr * per;
      const int q0 = pr * 2 * s, q1 = q0 + s;
      const int i0 = 4 * (u / (s / 4)), j0 = 4 * (u % (s / 4));
      float acc[4][4] = {};
      for (int k = j0; k < s; ++k) {  // inv(L) block is lower: rows k >= j0 only
        const float4 av = make_float4(S[(q1 + i0) * SLD + q0 + k], S[(q1 + i0 + 1) * SLD + q0 + k],
                                      S[(q1 + i0 + 2) * SLD + q0 + k],
                                      S[(q1 + i0 + 3) * SLD + q0 + k]);
        fma4x4(acc, av, *reinterpret_cast<const float4*>(Xs + (q0 + k) * SLD + q0 + j0));
      }
      float* T = Tm + pr * s * (s + 4);
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4*>(T + (i0 + x) * (s + 4) + j0) =
            make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
    }
    __syncthreads();
    for (int t = tid; t < per * npair; t += CI_THREADS) {
      const int pr = t / per, u = t - pr * per;
      const int q0 = pr * 2 * s, q1 = q0 + s;
      const int i0 = 4 * (u / (s / 4)), j0 = 4 * (u % (s / 4));
      const float* T = Tm + pr * s * (s + 4);
      float acc[4][4] = {};
      for (int k = 0; k <= i0 + 3; ++k) {  // inv(L) block is lower: columns k <= row
        const float4 av =
            make_float4(Xs[(q1 + i0) * SLD + q1 + k], Xs[(q1 + i0 + 1) * SLD + q1 + k],
                        Xs[(q1 + i0 + 2) * SLD + q1 + k], Xs[(q1 + i0 + 3) * SLD + q1 + k]);
        fma4x4(acc, av, *reinterpret_cast<const float4*>(T + k * (s + 4) + j0));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
        *reinterpret_cast<float4*>(Xs + (q1 + i0 + x) * SLD + q0 + j0) =
            make_float4(-acc[x][0], -acc[x][1], -acc[x][2], -acc[x][3]);
    }
    __syncthreads();
  }

  for (int i = warp; i < nb; i += CI_WARPS) {
    for (int j = lane; j < nb; j += 32) {
      if (j <= i) P[(o + i) * ld + (o + j)] = S[i * SLD + j];
      X[(o + i) * ld + (o + j)] = (j <= i) ? Xs[i * SLD + j] : 0.f;
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

// Same, four columns per thread (in % 4 == 0): U[i][k..k+3] is the float4 of
// row in-1-i of X that starts at column in-4-k, reversed.  Only the upper part
// of X's row is read.
__global__ void extract_u_vec_kernel(const float* X, int64_t in, float* U) {
  const int64_t in4 = in >> 2;
  for (int64_t i = blockIdx.y; i < in; i += gridDim.y) {
    const float* src = X + (in - 1 - i) * in;
    float4* dst = reinterpret_cast<float4*>(U + i * in);
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < in4;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t k = 4 * t;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k + 3 >= i) {
        const float4 v = *reinterpret_cast<const float4*>(src + (in - 4 - k));
        o = make_float4(k >= i ? v.w : 0.f, k + 1 >= i ? v.z : 0.f, k + 2 >= i ? v.y : 0.f, v.x);
      }
      dst[t] = o;
    }
  }
}

// rank of each column by decreasing sumsq (exact FP64 column sums of squares,
// i.e. diag(X^T X)); equal values keep index order.
// A NaN key (NaN or infinite inputs) ranks as -inf, so that (key, index) stays
// a strict total order and perm is always a permutation of 0..in-1.
__device__ __forceinline__ double rank_key(double x) {
  return x == x ? x : __longlong_as_double(static_cast<long long>(0xfff0000000000000ULL));
}

__global__ void act_order_rank_kernel(const double* d, int64_t in, int32_t* perm,
                                      int32_t* invperm) {
  __shared__ double tile[1024];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const double di = i < in ? rank_key(d[i]) : 0.0;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < in; j0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x)
      tile[t] = (j0 + t < in) ? rank_key(d[j0 + t]) : 0.0;
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

constexpr int kCholSmem = (2 * NB * SLD + SP * SLD + 64 * TLD + NB + 2 * SP) * sizeof(float);

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
  if (!launch_ok()) return PIQ_ERR_CUDA;

  // 3. Cholesky, panel by panel; diagonal inverses land in X
  for (int64_t k0 = 0; k0 < in; k0 += NB) {
    const int nb = static_cast<int>(std::min<int64_t>(NB, in - k0));
    const int nbp = nb <= 32 ? 32 : (nb <= 64 ? 64 : 128);
    note_launch();
    if (launch_pdl(chol_inv_kernel, dim3(1), dim3(CI_THREADS), kCholSmem, stream, P, X, ld, k0,
                   nb, nbp, st) != cudaSuccess)
      return PIQ_ERR_CUDA;
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
    const bool vec = in % 4 == 0 && (reinterpret_cast<uintptr_t>(X) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(U) & 15u) == 0;
    const int64_t cols = vec ? in / 4 : in;
    dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(cols, 256), 64)),
              static_cast<unsigned>(std::min<int64_t>(in, 65535)));
    note_launch();
    if (vec)
      extract_u_vec_kernel<<<grid, 256, 0, stream>>>(X, in, U);
    else
      extract_u_kernel<<<grid, 256, 0, stream>>>(X, in, U);
  }
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

int launch_act_order_perm(const double* sumsq, int64_t in, int32_t* perm, int32_t* invperm,
                          cudaStream_t stream) {
  note_launch();
  act_order_rank_kernel<<<static_cast<unsigned>(ceil_div(in, 256)), 256, 0, stream>>>(
      sumsq, in, perm, invperm);
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

int launch_identity_perm(int64_t in, int32_t* perm, int32_t* invperm, cudaStream_t stream) {
  note_launch();
  identity_perm_kernel<<<static_cast<unsigned>(ceil_div(in, 256)), 256, 0, stream>>>(in, perm,
                                                                                     invperm);
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace piq
