// GPTQ column sweep in FP64 on the Cholesky factor R of the damped Hessian.
//
// "GPTQ versus AWQ objectives", section "A strong answer", listing loop body:
// at each group start (j % g == 0) a per-row scale max|W[:, j:j+g]| / qmax from
// the current, already updated W; Q[:, j] = clip(round(W[:, j] / scale),
// -qmax-1, qmax) * scale; err = (W[:, j] - Q[:, j]) / U[j, j]; every later column
// gets W[:, k] -= err * U[j, k] (U = cholesky(inv(H_d)).T).  The remark after
// the listing batches the updates over column blocks so they run as GEMMs.
//
// Exact reformulation used here (no inverse of H_d is formed).  With H_d =
// R R^T, R = inv(U) upper triangular (factor64.cu), the listing's updates obey
// W0 - Q = U^T err, i.e. err = R^T (W0 - Q) row by row.  Hence, at the start of
// a block of columns G = [b, e), the current weights are
//     W_G = W0_G + acc_G inv(R_GG),   acc = sum over earlier columns p of
//                                           (W0[:, p] - Q[:, p]) R[p, :]
// and inside the block the listing's loop runs unchanged with inv(R_GG), which
// is the diagonal block U_GG of U.  After the block one product
//     acc[:, e:] += (W0 - Q)[:, G] R[G, e:]
// carries its rounding errors to every later column.  The original weights
// W0 are never modified; acc (fp64) collects the updates.  A group that
// starts at a block start and ends past the block takes its scale from
// W0_G + acc_G inv(R_GG) over the whole group (group_scale64_kernel).
//
// Everything is FP64: the in-block loop, the block-start weights, and the
// update product (FP64-grade on the INT8 tensor cores, ozaki.cu).  At a
// 28672-column layer, FP32 arithmetic in any of these moves w/scale by 1e-6 to
// 1e-5, enough to flip thousands of rounding decisions against the FP64
// evaluation of the same loop; FP64 brings that below 1e-9.
//
// Kernel: 64 rows per CTA (the fp64 row state and the 128 x 128 fp64 U_GG fill
// shared memory), 256 threads for the loads and the block-start product, one
// thread per row for the serial column loop (32-column register windows, the
// pending in-window updates subtracted where a group start inside the block
// reads later columns).  Rounding: IEEE division and rint (half to even), the
// listing's np.round of the true quotient W / scale.
#include <algorithm>
#include <vector>

#include "internal.h"

namespace piq {

namespace {

constexpr int B = kSweepB;   // 128
constexpr int RS = 64;       // rows per CTA
constexpr int SUB = 32;      // columns per register window
constexpr int THREADS = 256;
constexpr int LDW = B + 1;   // fp64 row-state stride
constexpr int kSmem = B * B * 8 + RS * LDW * 8 + B * 8 + 64;
constexpr int CST = B + 4;   // code row stride in bytes (rows in distinct banks)
constexpr int kSmemQ = B * B * 8 + RS * LDW * 8 + B * 8 + 10 * RS * 8 + RS * CST;
constexpr int64_t kSuperBlock = 1024;  // columns per superblock of the block updates

// rint(w / scale) for the IEEE quotient, from w * (1 / scale): the product is
// within a few units in the last place of the quotient, so it can only round
// differently within ~1e-12 |w / scale| of a half-integer, where the division
// itself decides (rare, out of line).
__device__ __noinline__ double code64_by_division(double w, double scale) {
  return rint(w / scale);
}
__device__ __forceinline__ double code64(double w, double scale, double rscale) {
  const double t = w * rscale;
  const double q = rint(t);
  return fabs(fabs(t - q) - 0.5) < 1e-12 * fmax(1.0, fabs(t)) ? code64_by_division(w, scale) : q;
}

// 2^e for |e| well inside the normal range, from the exponent field.
__device__ __forceinline__ double pow2(int e) {
  return __longlong_as_double(static_cast<long long>(1023 + e) << 52);
}

struct Row64 {
  double scale, rscale, cmin, cmax, fqmax;
  int64_t next_gs, b, in, g, ngroups, row;
  int kb;
  bool valid;
};

// Scale (and zero-point) of a group from the extremes of its current weights:
// symmetric m = max |w|; asymmetric m = max(0, max w), mn = min(0, min w).
__device__ __forceinline__ void set_group(double m, double mn, bool asym, Row64& st,
                                          float* __restrict__ qscale, uint8_t* __restrict__ qzero,
                                          int64_t grp) {
  if (!asym) {
    st.scale = m / st.fqmax;
  } else {
    st.scale = (m - mn) / st.fqmax;
    double z = st.scale > 0.0 ? rint(-mn / st.scale) : 0.0;
    z = fmin(fmax(z, 0.0), st.fqmax);
    st.cmin = -z;
    st.cmax = st.fqmax - z;
    if (st.valid) qzero[st.row * st.ngroups + grp] = static_cast<uint8_t>(z);
  }
  st.rscale = st.scale > 0.0 ? 1.0 / st.scale : 0.0;
  if (st.valid) qscale[st.row * st.ngroups + grp] = static_cast<float>(st.scale);
}

__global__ void __launch_bounds__(THREADS, 1)
    sweep64_kernel(const float* __restrict__ W0, const double* __restrict__ acc, int64_t out,
                   int64_t in, const double* __restrict__ Ub, int64_t b, int kb, int bits, int g,
                   int scale_given, int8_t* __restrict__ codes, float* __restrict__ qscale,
                   uint8_t* __restrict__ qzero, int8_t* __restrict__ dq, int* __restrict__ dex,
                   int64_t dkpad, int ds, double* __restrict__ dsb, int64_t ldsb,
                   DeviceStatus* st) {
  extern __shared__ __align__(16) double smem64[];
  double* Us = smem64;             // [B][B] U_GG
  double* Wr = Us + B * B;         // [RS][LDW] row state, then W0 - Q of used columns
  double* inv_u = Wr + RS * LDW;   // [B] 1 / U_jj
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  if (status_bad(st)) return;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * RS;
  const int rows_here = static_cast<int>(std::min<int64_t>(RS, out - row0));
  for (int idx = tid; idx < B * B; idx += THREADS) Us[idx] = Ub[idx];
  for (int j = tid; j < B; j += THREADS) inv_u[j] = j < kb ? 1.0 / Ub[j * B + j] : 0.0;
  for (int idx = tid; idx < RS * B; idx += THREADS) {
    const int r = idx >> 7, c = idx & (B - 1);
    Wr[r * LDW + c] = (r < rows_here && c < kb) ? acc[(row0 + r) * in + b + c] : 0.0;
  }
  __syncthreads();
  // W_G = W0_G + acc_G U_GG: thread (ty, tx) owns rows 4 ty .. + 3, columns tx + 16 c
  {
    const int ty = tid >> 4, tx = tid & 15;
    double o[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 8; ++c) o[i][c] = 0.0;
    for (int k = 0; k < kb; ++k) {
      double a[4], u[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Wr[(4 * ty + i) * LDW + k];
#pragma unroll
      for (int c = 0; c < 8; ++c) u[c] = Us[k * B + tx + 16 * c];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 8; ++c) o[i][c] = fma(a[i], u[c], o[i][c]);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 4 * ty + i;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int col = tx + 16 * c;
        double w = 0.0;
        if (r < rows_here && col < kb)
          w = static_cast<double>(W0[(row0 + r) * in + b + col]) + o[i][c];
        Wr[r * LDW + col] = w;
      }
    }
  }
  __syncthreads();

  if (tid < RS) {
    const bool asym = qzero != nullptr;
    Row64 rs;
    const int qmax = (1 << (bits - 1)) - 1;
    rs.fqmax = asym ? static_cast<double>((1 << bits) - 1) : static_cast<double>(qmax);
    rs.cmin = -static_cast<double>(qmax) - 1.0;
    rs.cmax = static_cast<double>(qmax);
    rs.kb = kb;
    rs.b = b;
    rs.in = in;
    rs.g = g;
    rs.ngroups = (in + g - 1) / g;
    rs.row = row0 + tid;
    rs.valid = tid < rows_here;
    rs.scale = 0.0;
    // the block's first column: a group that continues from an earlier block,
    // or one whose scale was taken over its whole width beforehand, keeps the
    // stored scale; otherwise it is computed at column 0 below
    const int64_t boff = b % g;
    if (boff != 0 || scale_given) {
      const int64_t grp = b / g;
      rs.scale = rs.valid ? static_cast<double>(qscale[rs.row * rs.ngroups + grp]) : 0.0;
      if (asym) {
        const double z = rs.valid ? static_cast<double>(qzero[rs.row * rs.ngroups + grp]) : 0.0;
        rs.cmin = -z;
        rs.cmax = rs.fqmax - z;
      }
      rs.next_gs = (boff == 0) ? g : g - boff;
    } else {
      rs.next_gs = 0;
    }
    rs.rscale = rs.scale > 0.0 ? 1.0 / rs.scale : 0.0;
    double* wrow = Wr + tid * LDW;
    const float* w0row = W0 + rs.row * in + b;
    int8_t* crow = codes + rs.row * in + b;
    for (int c0 = 0; c0 < kb; c0 += SUB) {
      double ws[SUB], e[SUB];
#pragma unroll
      for (int k = 0; k < SUB; ++k) {
        ws[k] = wrow[c0 + k];
        e[k] = 0.0;
      }
#pragma unroll
      for (int jj = 0; jj < SUB; ++jj) {
        const int j = c0 + jj;
        if (j < kb) {
          if (j == rs.next_gs) {
            // group start inside the block: its whole group lies in the block
            const int jend = static_cast<int>(std::min<int64_t>(j + g, kb));
            double m = 0.0, mn = 0.0;
#pragma unroll
            for (int k = 0; k < SUB; ++k)
              if (k >= jj && c0 + k < jend) {
                m = fmax(m, asym ? ws[k] : fabs(ws[k]));
                mn = fmin(mn, ws[k]);
              }
            for (int c = c0 + SUB; c < jend; ++c) {
              double v = wrow[c];
#pragma unroll
              for (int p = 0; p < SUB; ++p)
                if (p < jj) v = fma(-e[p], Us[(c0 + p) * B + c], v);
              m = fmax(m, asym ? v : fabs(v));
              mn = fmin(mn, v);
            }
            set_group(m, mn, asym, rs, qscale, qzero, (b + j) / g);
            rs.next_gs += g;
          }
          const double wj = ws[jj];
          const double sc = rs.scale;
          const double qv = sc > 0.0 ? fmin(fmax(code64(wj, sc, rs.rscale), rs.cmin), rs.cmax)
                                     : 0.0;
          const double err = (wj - qv * sc) * inv_u[j];
          e[jj] = err;
          if (rs.valid) crow[j] = static_cast<int8_t>(qv);
          // W0 - Q of this column replaces its slot in the row state
          wrow[j] = rs.valid ? static_cast<double>(w0row[j]) - qv * sc : 0.0;
#pragma unroll
          for (int k = jj + 1; k < SUB; ++k) ws[k] = fma(-err, Us[j * B + c0 + k], ws[k]);
        }
      }
      // the window's errors update every later column of the block
      for (int c = c0 + SUB; c < kb; ++c) {
        double v = wrow[c];
#pragma unroll
        for (int p = 0; p < SUB; ++p) v = fma(-e[p], Us[(c0 + p) * B + c], v);
        wrow[c] = v;
      }
    }
    // this row's W0 - Q in fp64 for the superblock's product (when one is kept)
    if (dsb != nullptr && rs.valid) {
      double* drow = dsb + rs.row * ldsb;
      for (int c = 0; c < kb; ++c) drow[c] = wrow[c];
    }
    // digits of this row's W0 - Q for the block's own update product (ozaki.cu layout)
    double m = 0.0;
    for (int c = 0; c < kb; ++c) m = fmax(m, fabs(wrow[c]));
    int ex = 0;
    if (m > 0.0) frexp(m, &ex);
    if (rs.valid) {
      dex[rs.row] = ex;
      const int64_t plane = out * dkpad;
      for (int c4 = 0; c4 < dkpad; c4 += 4) {
        double y[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int c = c4 + t;
          y[t] = (c < kb && m > 0.0) ? wrow[c] * pow2(6 - ex) : 0.0;
        }
#pragma unroll
        for (int i = 0; i < kMaxDigits; ++i) {
          if (i < ds) {
            uint32_t w = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const double di = rint(y[t]);
              y[t] = (y[t] - di) * 128.0;
              w |= (static_cast<uint32_t>(static_cast<int>(di)) & 0xFFu) << (8 * t);
            }
            *reinterpret_cast<uint32_t*>(dq + i * plane + rs.row * dkpad + c4) = w;
          }
        }
      }
    }
  }
}

// The same block for g % 128 == 0 (no group starts inside the block except at
// its first column).  256 threads, 64 rows, in five steps:
//  1. asynchronous copies: U_GG (128 KB) and the rows' acc_G into shared memory;
//  2. W_G = W0_G + acc_G U_GG: U_GG is upper triangular, so column c sums over
//     k <= c; warp w owns the column quads {w, 15-w, 16+w, 31-w} (equal work)
//     and lane l the rows l and l+32;
//  3. the row scale from the maxima of the four 32-column windows;
//  4. the serial column loop: warp w owns rows 32 (w % 2) .. + 31 (one per
//     lane) and window q = w / 2 (block columns 32 q .. 32 q + 31) in
//     registers.  Phase p (0..3): the window-p threads apply window p-1's
//     errors to their window and run its serial loop; the threads of later
//     windows apply the same errors meanwhile.  The rounding takes w * (1 / s)
//     and only records whether the product came within 1e-12 of a half
//     integer; a thread that saw one re-runs its window from the saved state
//     with the exact quotient there (code64), which gives what the plain loop
//     gives;
//  5. write-out, one warp per row at a time (lane l: columns 4l .. 4l+3):
//     codes, W0 - Q, its digits and exponent.
constexpr int QT = 256;

// The serial loop of one window in shared memory with code64 rounding (the
// rare path): wrow holds the window's state at the start of the loop and gets
// its errors; crow gets its codes.
__device__ __noinline__ void window_redo64(double* wrow, const double* Us, const double* inv_u,
                                           int c0, int kb, double sc, double rsc, double cmin,
                                           double cmax, int8_t* crow) {
  for (int jj = 0; jj < SUB; ++jj) {
    const int j = c0 + jj;
    if (j >= kb) break;
    const double wj = wrow[j];
    const double qv = sc > 0.0 ? fmin(fmax(code64(wj, sc, rsc), cmin), cmax) : 0.0;
    const double err = (wj - qv * sc) * inv_u[j];
    crow[j] = static_cast<int8_t>(qv);
    wrow[j] = err;
    for (int k = jj + 1; k < SUB; ++k) wrow[c0 + k] = fma(-err, Us[j * B + c0 + k], wrow[c0 + k]);
  }
}

__global__ void __launch_bounds__(QT, 1)
    sweep64q_kernel(const float* __restrict__ W0, const double* __restrict__ acc, int64_t out,
                    int64_t in, const double* __restrict__ Ub, int64_t b, int kb, int bits,
                    int g, int scale_given, int8_t* __restrict__ codes,
                    float* __restrict__ qscale, uint8_t* __restrict__ qzero,
                    int8_t* __restrict__ dq, int* __restrict__ dex, int64_t dkpad, int ds,
                    double* __restrict__ dsb, int64_t ldsb, DeviceStatus* st) {
  extern __shared__ __align__(16) double smem64[];
  double* Us = smem64;                                   // [B][B] U_GG
  double* Wr = Us + B * B;                               // [RS][LDW] row state / errors
  double* inv_u = Wr + RS * LDW;                         // [B]
  double* scale_s = inv_u + B;                           // [RS]
  double* zero_s = scale_s + RS;                         // [RS]
  double* mx = zero_s + RS;                              // [4][RS] window maxima
  double* mn = mx + 4 * RS;                              // [4][RS] window minima
  int8_t* Cs = reinterpret_cast<int8_t*>(mn + 4 * RS);   // [RS][CST] codes
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  pdl_wait();
  if (status_bad(st)) return;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * RS;
  const int rows_here = static_cast<int>(std::min<int64_t>(RS, out - row0));

  // ---- 1. loads
  for (int idx = tid; idx < B * B / 2; idx += QT) cp_async16(Us + 2 * idx, Ub + 2 * idx);
  for (int idx = tid; idx < RS * B; idx += QT) {
    const int r = idx >> 7, c = idx & (B - 1);
    if (r < rows_here && c < kb)
      cp_async8(Wr + r * LDW + c, acc + (row0 + r) * in + b + c);
    else
      Wr[r * LDW + c] = 0.0;
  }
  cp_async_wait_all();
  __syncthreads();
  if (tid < B) inv_u[tid] = tid < kb ? 1.0 / Us[tid * B + tid] : 0.0;

  // ---- 2. W_G = W0_G + acc_G U_GG (k <= c)
  {
    const int qd[4] = {warp, 15 - warp, 16 + warp, 31 - warp};  // ascending
    double o[2][4][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[h][s][c] = 0.0;
    const double* wa = Wr + lane * LDW;
    const double* wb = Wr + (lane + 32) * LDW;
    int k = 0;
#pragma unroll
    for (int s0 = 0; s0 < 4; ++s0) {  // quads s0..3 still take k
      const int kend = 4 * qd[s0] + 4;
#pragma unroll 4
      for (; k < kend; ++k) {
        const double a0 = wa[k], a1 = wb[k];
        const double* urow = Us + k * B;
#pragma unroll
        for (int s = s0; s < 4; ++s) {
          const double2 u01 = *reinterpret_cast<const double2*>(urow + 4 * qd[s]);
          const double2 u23 = *reinterpret_cast<const double2*>(urow + 4 * qd[s] + 2);
          const double u[4] = {u01.x, u01.y, u23.x, u23.y};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            o[0][s][c] = fma(a0, u[c], o[0][s][c]);
            o[1][s][c] = fma(a1, u[c], o[1][s][c]);
          }
        }
      }
    }
    __syncthreads();  // every read of acc_G is done
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      const bool rv = r < rows_here;
      const float* w0r = W0 + (row0 + r) * in + b;
#pragma unroll
      for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = 4 * qd[s] + c;
          Wr[r * LDW + col] =
              (rv && col < kb) ? static_cast<double>(w0r[col]) + o[h][s][c] : 0.0;
        }
    }
  }
  __syncthreads();

  // ---- 3. the row scale
  const bool asym = qzero != nullptr;
  const int qmax = (1 << (bits - 1)) - 1;
  const double fqmax = asym ? static_cast<double>((1 << bits) - 1) : static_cast<double>(qmax);
  const int64_t ngroups = (in + g - 1) / g;
  const int q = warp >> 1;                  // window
  const int lrow = (warp & 1) * 32 + lane;  // row within the CTA
  const int64_t row = row0 + lrow;
  const bool valid = lrow < rows_here;
  double* wrow = Wr + lrow * LDW;
  const int c0 = SUB * q;
  double ws[SUB];
  {
    double m = 0.0, m2 = 0.0;
#pragma unroll
    for (int k = 0; k < SUB; ++k) {
      ws[k] = wrow[c0 + k];  // zero past kb
      m = fmax(m, asym ? ws[k] : fabs(ws[k]));
      m2 = fmin(m2, ws[k]);
    }
    mx[q * RS + lrow] = m;
    mn[q * RS + lrow] = m2;
  }
  __syncthreads();
  if (q == 0) {
    // a group starts here (its whole width is this block when g == 128)
    // unless its scale was taken beforehand, or it continues from earlier
    double sc, z = 0.0;
    if (b % g == 0 && !scale_given) {
      const double m = fmax(fmax(mx[lrow], mx[RS + lrow]), fmax(mx[2 * RS + lrow], mx[3 * RS + lrow]));
      const double m2 = fmin(fmin(mn[lrow], mn[RS + lrow]), fmin(mn[2 * RS + lrow], mn[3 * RS + lrow]));
      if (!asym) {
        sc = m / fqmax;
      } else {
        sc = (m - m2) / fqmax;
        z = sc > 0.0 ? rint(-m2 / sc) : 0.0;
        z = fmin(fmax(z, 0.0), fqmax);
        if (valid) qzero[row * ngroups + b / g] = static_cast<uint8_t>(z);
      }
      if (valid) qscale[row * ngroups + b / g] = static_cast<float>(sc);
    } else {
      sc = valid ? static_cast<double>(qscale[row * ngroups + b / g]) : 0.0;
      if (asym && valid) z = static_cast<double>(qzero[row * ngroups + b / g]);
    }
    scale_s[lrow] = sc;
    zero_s[lrow] = z;
  }
  __syncthreads();

  // ---- 4. the serial column loop
  {
    const double sc = scale_s[lrow];
    const double rsc = sc > 0.0 ? 1.0 / sc : 0.0;
    const double cmin = asym ? -zero_s[lrow] : -static_cast<double>(qmax) - 1.0;
    const double cmax = asym ? fqmax - zero_s[lrow] : static_cast<double>(qmax);
    int8_t* crow = Cs + lrow * CST;
    for (int p = 0; p < 4; ++p) {
      if (q >= p && SUB * p < kb) {
        if (p > 0) {
          const int cp = SUB * (p - 1);
#pragma unroll 4
          for (int t = 0; t < SUB; ++t) {
            const double ev = wrow[cp + t];
            const double* urow = Us + (cp + t) * B + c0;
#pragma unroll
            for (int k = 0; k < SUB; ++k) ws[k] = fma(-ev, urow[k], ws[k]);
          }
        }
        if (q == p) {
#pragma unroll
          for (int k = 0; k < SUB; ++k) wrow[c0 + k] = ws[k];  // the state, for a redo
          bool near = false;
#pragma unroll
          for (int jj = 0; jj < SUB; ++jj) {
            const int j = c0 + jj;
            if (j < kb) {
              const double wj = ws[jj];
              const double t = wj * rsc;
              const double r = rint(t);
              near |= fabs(fabs(t - r) - 0.5) < 1e-12 * fmax(1.0, fabs(t));
              const double qv = sc > 0.0 ? fmin(fmax(r, cmin), cmax) : 0.0;
              const double err = (wj - qv * sc) * inv_u[j];
              crow[j] = static_cast<int8_t>(qv);
              ws[jj] = err;
#pragma unroll
              for (int k = jj + 1; k < SUB; ++k) ws[k] = fma(-err, Us[j * B + c0 + k], ws[k]);
            }
          }
          if (near) {
            window_redo64(wrow, Us, inv_u, c0, kb, sc, rsc, cmin, cmax, crow);
          } else {
#pragma unroll
            for (int k = 0; k < SUB; ++k) wrow[c0 + k] = ws[k];
          }
        }
      }
      __syncthreads();
    }
  }

  // ---- 5. write-out: warp w takes rows w, w+8, ...; lane l columns 4l .. 4l+3
  const int64_t plane = out * dkpad;
  const bool c4_aligned = ((in | b) & 3) == 0 && (reinterpret_cast<uintptr_t>(codes) & 3) == 0;
  for (int r = warp; r < rows_here; r += QT / 32) {
    const int64_t grow = row0 + r;
    const double sc = scale_s[r];
    const float* w0r = W0 + grow * in + b;
    const int8_t* cr = Cs + r * CST;
    double d[4];
    double m = 0.0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = 4 * lane + t;
      d[t] = c < kb ? static_cast<double>(w0r[c]) - static_cast<double>(cr[c]) * sc : 0.0;
      m = fmax(m, fabs(d[t]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    int8_t* cg = codes + grow * in + b;
    if (c4_aligned && 4 * lane + 3 < kb) {
      *reinterpret_cast<uint32_t*>(cg + 4 * lane) = *reinterpret_cast<const uint32_t*>(cr + 4 * lane);
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (4 * lane + t < kb) cg[4 * lane + t] = cr[4 * lane + t];
    }
    if (dsb != nullptr) {
      double* drow = dsb + grow * ldsb;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (4 * lane + t < kb) drow[4 * lane + t] = d[t];
    }
    int ex = 0;
    if (m > 0.0) frexp(m, &ex);
    if (lane == 0) dex[grow] = ex;
    if (4 * lane < dkpad) {
      const double sc6 = m > 0.0 ? pow2(6 - ex) : 0.0;
      double y[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) y[t] = d[t] * sc6;
#pragma unroll
      for (int i = 0; i < kMaxDigits; ++i) {
        if (i < ds) {
          uint32_t w = 0;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const double di = rint(y[t]);
            y[t] = (y[t] - di) * 128.0;
            w |= (static_cast<uint32_t>(static_cast<int>(di)) & 0xFFu) << (8 * t);
          }
          *reinterpret_cast<uint32_t*>(dq + i * plane + grow * dkpad + 4 * lane) = w;
        }
      }
    }
  }
}

// Scale (and zero-point) of the group starting at column b and ending at gend
// past the current block, from its current weights W0_G + acc_G inv(R_GG):
// one thread per row solves y R_GG = acc_G by forward substitution in FP64
// (R[i][k] = L[in-1-i][in-1-k]).
__global__ void group_scale64_kernel(const float* __restrict__ W0, const double* __restrict__ acc,
                                     int64_t out, int64_t in, const double* __restrict__ L,
                                     int64_t b, int64_t gend, int bits, int g,
                                     float* __restrict__ qscale, uint8_t* __restrict__ qzero,
                                     double* __restrict__ yscr, DeviceStatus* st) {
  pdl_launch_dependents();
  pdl_wait();
  if (status_bad(st)) return;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= out) return;
  const int64_t gw = gend - b;
  double* y = yscr + r * gw;  // this row's solution, in place of acc_G
  const bool asym = qzero != nullptr;
  double m = 0.0, mn = 0.0;
  for (int64_t k = 0; k < gw; ++k) {
    double v = acc[r * in + b + k];
    for (int64_t p = 0; p < k; ++p) v = fma(-y[p], L[(in - 1 - b - p) * in + (in - 1 - b - k)], v);
    v /= L[(in - 1 - b - k) * in + (in - 1 - b - k)];
    y[k] = v;
    const double w = static_cast<double>(W0[r * in + b + k]) + v;
    m = fmax(m, asym ? w : fabs(w));
    mn = fmin(mn, w);
  }
  const int64_t ngroups = (in + g - 1) / g;
  const int qmax = (1 << (bits - 1)) - 1;
  const double fq = asym ? static_cast<double>((1 << bits) - 1) : static_cast<double>(qmax);
  double sc;
  if (!asym) {
    sc = m / fq;
  } else {
    sc = (m - mn) / fq;
    double z = sc > 0.0 ? rint(-mn / sc) : 0.0;
    z = fmin(fmax(z, 0.0), fq);
    qzero[r * ngroups + b / g] = static_cast<uint8_t>(z);
  }
  qscale[r * ngroups + b / g] = static_cast<float>(sc);
}

}  // namespace

// Column blocks of width <= 128 where each group start inside a block has its
// whole group inside that block (the same cut as the FP32 sweep).
static void block_partition64(int64_t in, int g, std::vector<int64_t>* starts) {
  starts->clear();
  int64_t b = 0;
  while (b < in) {
    starts->push_back(b);
    int64_t e = std::min<int64_t>(b + B, in);
    for (int64_t s = (b / g + 1) * g; s < e; s += g) {
      if (std::min<int64_t>(s + g, in) > e) {
        e = s;
        break;
      }
    }
    b = e;
  }
  starts->push_back(in);
}

int sweep64_blocks(int64_t in, int g) {
  std::vector<int64_t> s;
  block_partition64(in, g, &s);
  return static_cast<int>(s.size()) - 1;
}

int64_t sweep64_workspace_bytes(int64_t out, int64_t in, int g) {
  Sweep64Ws w;
  return carve_sweep64(nullptr, out, in, g, &w);
}

int64_t carve_sweep64(void* base, int64_t out, int64_t in, int g, Sweep64Ws* w) {
  uint8_t* p0 = static_cast<uint8_t*>(base);
  int64_t off = 0;
  auto take = [&](int64_t bytes) -> uint8_t* {
    off = (off + 255) / 256 * 256;
    uint8_t* p = p0 ? p0 + off : nullptr;
    off += std::max<int64_t>(bytes, 1);
    return p;
  };
  const int nblk = sweep64_blocks(in, g);
  const int64_t kpad = digit_kpad(B);
  w->nblocks = nblk;
  w->acc = reinterpret_cast<double*>(take(out * in * 8));
  w->Ub = reinterpret_cast<double*>(take(static_cast<int64_t>(nblk) * B * B * 8));
  w->starts = reinterpret_cast<int64_t*>(take((nblk + 1) * 8));
  w->dq = reinterpret_cast<int8_t*>(take(static_cast<int64_t>(kSweepDigits) * out * kpad));
  w->dex = reinterpret_cast<int*>(take(out * 4));
  w->rq = reinterpret_cast<int8_t*>(take(static_cast<int64_t>(kSweepDigits) * in * kpad));
  w->rex = reinterpret_cast<int*>(take(in * 4));
  // group scales over more than one block: one row's solution of the group width
  const int64_t gw = g > B ? std::min<int64_t>(g, in) : 0;
  w->yscr = reinterpret_cast<double*>(take(out * gw * 8));
  // superblocks (g <= 128 only): W0 - Q of the superblock in fp64 and the
  // digits of the superblock's product
  const int64_t sbw = (g <= B) ? std::min<int64_t>(kSuperBlock, in) : 0;
  const int64_t sbk = sbw ? digit_kpad(sbw) : 0;
  w->dsb = reinterpret_cast<double*>(take(out * sbw * 8));
  w->sbq = reinterpret_cast<int8_t*>(take(static_cast<int64_t>(kSweepDigits) * out * sbk));
  w->sbex = reinterpret_cast<int*>(take(out * 4));
  w->sbrq = reinterpret_cast<int8_t*>(take(static_cast<int64_t>(kSweepDigits) * in * sbk));
  w->sbrex = reinterpret_cast<int*>(take(in * 4));
  return (off + 255) / 256 * 256;
}

int run_gptq_sweep64(const float* W0, int64_t out, int64_t in, const double* L, int bits, int g,
                     int8_t* codes, float* qscale, uint8_t* qzero, const Sweep64Ws& w,
                     DeviceStatus* st, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(sweep64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmem) != cudaSuccess ||
        cudaFuncSetAttribute(sweep64q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemQ) != cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  std::vector<int64_t> starts;
  block_partition64(in, g, &starts);
  const int nblk = static_cast<int>(starts.size()) - 1;
  if (nblk != w.nblocks) return PIQ_ERR_INVALID_ARG;
  int rc = cuda_rc(cudaMemcpyAsync(w.starts, starts.data(), sizeof(int64_t) * starts.size(),
                                   cudaMemcpyHostToDevice, stream));
  if (rc != PIQ_OK) return rc;
  rc = cuda_rc(cudaMemsetAsync(w.acc, 0, sizeof(double) * out * in, stream));
  if (rc != PIQ_OK) return rc;
  rc = launch_block_inverses(L, in, w.starts, nblk, w.Ub, stream);
  if (rc != PIQ_OK) return rc;
  const unsigned grid = static_cast<unsigned>(ceil_div(out, RS));
  // superblocks: runs of blocks of at most kSuperBlock columns.  Inside one, a
  // block's product updates only the superblock's later columns; the columns
  // past it get the whole superblock's product at once.  Only when every group
  // lies inside a block (g <= 128): a group that starts at a block start and
  // runs past it reads acc past the block, which must then be complete.
  const bool use_sb = g <= B;
  int bi = 0;
  while (bi < nblk) {
    const int64_t S0 = starts[bi];
    int bj = bi + 1;
    if (use_sb)
      while (bj < nblk && starts[bj + 1] - S0 <= kSuperBlock) ++bj;
    const int64_t S1 = use_sb ? starts[bj] : in;  // columns the blocks update directly
    for (int bk = bi; bk < bj; ++bk) {
      const int64_t b = starts[bk], e = starts[bk + 1];
      const int kb = static_cast<int>(e - b);
      const int64_t gend = std::min<int64_t>((b / g) * g + g, in);
      const bool wide = (b % g == 0) && gend > e;  // the group runs past this block
      if (wide) {
        note_launch();
        if (launch_pdl(group_scale64_kernel, dim3(static_cast<unsigned>(ceil_div(out, 128))),
                       dim3(128), 0, stream, W0, w.acc, out, in, L, b, gend, bits, g, qscale,
                       qzero, w.yscr, st) != cudaSuccess)
          return PIQ_ERR_CUDA;
      }
      DigitMat dA;
      dA.q = w.dq;
      dA.ex = w.dex;
      dA.rows = out;
      dA.kpad = digit_kpad(kb);
      dA.s = kSweepDigits;
      note_launch();
      const cudaError_t le =
          (g % B == 0)
              ? launch_pdl(sweep64q_kernel, dim3(grid), dim3(QT), kSmemQ, stream, W0, w.acc, out,
                           in, w.Ub + static_cast<int64_t>(bk) * B * B, b, kb, bits, g,
                           wide ? 1 : 0, codes, qscale, qzero, dA.q, dA.ex, dA.kpad, dA.s,
                           use_sb ? w.dsb + (b - S0) : nullptr,
                           static_cast<int64_t>(kSuperBlock), st)
              : launch_pdl(sweep64_kernel, dim3(grid), dim3(THREADS), kSmem, stream, W0, w.acc,
                           out, in, w.Ub + static_cast<int64_t>(bk) * B * B, b, kb, bits, g,
                           wide ? 1 : 0, codes, qscale, qzero, dA.q, dA.ex, dA.kpad, dA.s,
                           use_sb ? w.dsb + (b - S0) : nullptr,
                           static_cast<int64_t>(kSuperBlock), st);
      if (le != cudaSuccess) return PIQ_ERR_CUDA;
      const int64_t lim = use_sb ? S1 : in;
      if (e < lim) {
        // acc[:, e:lim] += (W0 - Q)[:, b:e] R[b:e, e:lim];  B operand row n, digit k:
        // R[b + k][e + n] = L[in-1-b-k][in-1-e-n], read from the mirror of L in
        // the upper triangle, P[in-1-e-n][in-1-b-k] (contiguous in k)
        DigitMat dB;
        dB.q = w.rq;
        dB.ex = w.rex;
        dB.rows = lim - e;
        dB.kpad = dA.kpad;
        dB.s = kSweepDigits;
        rc = launch_slice(L + (in - 1 - e) * in + (in - 1 - b), -in, -1, lim - e, kb,
                          kSweepDigits, &dB, stream);
        if (rc == PIQ_OK)
          rc = launch_ozaki_gemm(out, lim - e, dA, dB, 1.0, 1, 0, w.acc + e, in, st, stream);
        if (rc != PIQ_OK) return rc;
      }
    }
    if (use_sb && S1 < in) {
      // acc[:, S1:] += (W0 - Q)[:, S0:S1] R[S0:S1, S1:]
      const int64_t K = S1 - S0;
      DigitMat dA, dB;
      dA.q = w.sbq;
      dA.ex = w.sbex;
      dA.rows = out;
      dA.kpad = digit_kpad(K);
      dA.s = kSweepDigits;
      dB.q = w.sbrq;
      dB.ex = w.sbrex;
      dB.rows = in - S1;
      dB.kpad = dA.kpad;
      dB.s = kSweepDigits;
      rc = launch_slice(w.dsb, kSuperBlock, 1, out, K, kSweepDigits, &dA, stream);
      if (rc == PIQ_OK)
        rc = launch_slice(L + (in - 1 - S1) * in + (in - 1 - S0), -in, -1, in - S1, K,
                          kSweepDigits, &dB, stream);
      if (rc == PIQ_OK)
        rc = launch_ozaki_gemm(out, in - S1, dA, dB, 1.0, 1, 0, w.acc + S1, in, st, stream);
      if (rc != PIQ_OK) return rc;
    }
    bi = bj;
  }
  return PIQ_OK;
}

}  // namespace piq
