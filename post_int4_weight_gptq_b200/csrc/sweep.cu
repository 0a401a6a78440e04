// GPTQ column sweep, block by block.
//
// "GPTQ versus AWQ objectives", section "A strong answer", listing loop body:
// at each group start (j % g == 0) a per-row scale max|W[:, j:j+g]| / qmax from
// the current, already updated W; Q[:, j] = clip(round(W[:, j] / scale),
// -qmax-1, qmax) * scale; err = (W[:, j] - Q[:, j]) / U[j, j]; every later column
// gets W[:, k] -= err * U[j, k].  The remark after the listing batches the
// updates over column blocks: inside a block the updates are applied at once
// (here, in registers), and the block's errors update all later columns with
// one GEMM, W[:, e:] -= Err[:, b:e] U[b:e, e:] (FP32-accurate: three TF32
// tensor-core passes, tc_sgemm.cu; the SIMT kernel of simt_gemm.cu where the
// operands do not suit TMA).
//
// Blocks are at most 128 wide and are cut so that every group start is either
// a block start or has its whole group inside its block; a group scale then
// only reads columns whose updates are all applied (g | 128, 128 | g, or any
// other g), so the arithmetic is the listing's.
//
// Kernel layout: one thread per row (128 rows per CTA).  The row's block
// columns live in shared memory; a thread walks them in 32-column windows held
// in registers (the serial column loop with its in-window updates), then
// applies the window's errors to the later columns of the block.  The strictly
// upper part of U[b:e, b:e] sits in shared memory and is read by all lanes at
// the same address (broadcast).  The code stays small enough for the
// instruction cache: only the 32-column window is unrolled.  W/scale is an IEEE
// round-to-nearest division and rintf rounds half to even (the listing's
// np.round); the error uses the reciprocal of U[j, j].
//
// Asymmetric groups (qzero != NULL; a scale and zero-point per group, the
// uplatz.com report's Group Size paragraph, formula read as min/max affine
// rounding over a range widened to hold 0): at a group start
// scale = (max(0, max w) - min(0, min w)) / (2^bits - 1) and
// zero = rint(-min(0, min w) / scale); the signed code is clipped to
// [-zero, 2^bits - 1 - zero] instead of [-qmax - 1, qmax], and zero is stored as
// one byte per (row, group).  Everything else is the symmetric loop.
#include <algorithm>
#include <vector>

#include "internal.h"

namespace piq {

namespace {

constexpr int B = kSweepB;   // 128 block columns
constexpr int SUB = 32;      // columns per register window
constexpr int R = 128;       // rows per CTA, one per thread
constexpr int LDW = B + 4;   // row-state stride (float4-aligned, conflict-free per 8 lanes)
constexpr int LDC = B + 4;   // code staging row (bytes)
constexpr int kSweepSmem = B * B * 4 + B * 4 + R * LDW * 4 + R * LDC;
constexpr int kQuartersSmem = kSweepSmem + 2 * R * 4;

// Per-row state of the column loop.
struct SweepRow {
  float scale;
  float rscale;      // 1 / scale (0 when scale is 0)
  int64_t next_gs;   // block-relative column of the next group start
  float fqmax;       // qmax (symmetric) or 2^bits - 1 (asymmetric)
  float cmin, cmax;  // signed code range of the current group
  int kb;
  int64_t b, in, g, ngroups, row;
  bool valid;
};

// rint(w / scale) for the IEEE quotient, from w * (1 / scale): the product is
// within a few units in the last place of the quotient, so it can only round
// differently within ~1e-6 |w / scale| of a half-integer, where the division
// itself decides (rare, out of line).
__device__ __noinline__ float code_by_division(float w, float scale) {
  return rintf(__fdiv_rn(w, scale));
}
__device__ __forceinline__ float code_of(float w, float scale, float rscale) {
  const float t = w * rscale;
  const float q = rintf(t);
  return fabsf(fabsf(t - q) - 0.5f) < 1e-5f * fmaxf(1.f, fabsf(t)) ? code_by_division(w, scale)
                                                                   : q;
}

// Scale, zero-point and code range of an asymmetric group from the extremes of
// its current weights (mx = max(0, max w), mn = min(0, min w)).
__device__ __forceinline__ void asym_params(float mx, float mn, SweepRow& st,
                                            uint8_t* __restrict__ qzero, int64_t grp) {
  st.scale = __fdiv_rn(mx - mn, st.fqmax);
  float z = st.scale > 0.f ? rintf(__fdiv_rn(-mn, st.scale)) : 0.f;
  z = fminf(fmaxf(z, 0.f), st.fqmax);
  st.cmin = -z;
  st.cmax = st.fqmax - z;
  if (st.valid) qzero[st.row * st.ngroups + grp] = static_cast<uint8_t>(z);
}

// Group start at block column j (window base c0, jj = j - c0): the scale comes
// from the current weights of [j, j+g): the window in registers, later block
// columns in shared memory minus the updates still pending from window columns
// before j, and (only when j is the block start) columns past the block in W.
// Symmetric: m = max|w|.  Asymmetric: m = max(0, max w), mn = min(0, min w).
__device__ __forceinline__ void group_start(const float (&ws)[SUB], const float (&e)[SUB], int jj,
                                            int c0, SweepRow& st, const float* __restrict__ W,
                                            const float* Us, const float* wrow,
                                            float* __restrict__ qscale,
                                            uint8_t* __restrict__ qzero) {
  const int j = c0 + jj;
  const int64_t gend = std::min<int64_t>(st.b + j + st.g, st.in);
  const int jend = static_cast<int>(std::min<int64_t>(gend - st.b, st.kb));
  const bool asym = qzero != nullptr;
  float m = 0.f, mn = 0.f;
#pragma unroll
  for (int k = 0; k < SUB; ++k)
    if (k >= jj && c0 + k < jend) {
      m = fmaxf(m, asym ? ws[k] : fabsf(ws[k]));
      mn = fminf(mn, ws[k]);
    }
  for (int c = c0 + SUB; c < jend; ++c) {
    float v = wrow[c];
#pragma unroll
    for (int p = 0; p < SUB; ++p)
      if (p < jj) v = fmaf(-e[p], Us[(c0 + p) * B + c], v);
    m = fmaxf(m, asym ? v : fabsf(v));
    mn = fminf(mn, v);
  }
  if (gend > st.b + st.kb && st.valid) {
    const float* src = W + st.row * st.in;
    for (int64_t c = st.b + st.kb; c < gend; ++c) {
      m = fmaxf(m, asym ? src[c] : fabsf(src[c]));
      mn = fminf(mn, src[c]);
    }
  }
  const int64_t grp = (st.b + j) / st.g;
  if (asym)
    asym_params(m, mn, st, qzero, grp);
  else
    st.scale = __fdiv_rn(m, st.fqmax);
  st.rscale = st.scale > 0.f ? __frcp_rn(st.scale) : 0.f;
  if (st.valid) qscale[st.row * st.ngroups + grp] = st.scale;
  st.next_gs += st.g;
}

// Column c0 + JJ of the window, then the next: template recursion keeps every
// register index a compile-time constant.
template <bool GENERAL, int JJ>
__device__ __forceinline__ void sweep_col(float (&ws)[SUB], float (&e)[SUB], int c0, SweepRow& st,
                                          const float* __restrict__ W, const float* Us,
                                          const float* inv_u, const float* wrow, int8_t* code_row,
                                          float* __restrict__ qscale,
                                          uint8_t* __restrict__ qzero) {
  if constexpr (JJ < SUB) {
    const int j = c0 + JJ;
    if (j < st.kb) {
      if (GENERAL && j == st.next_gs)
        group_start(ws, e, JJ, c0, st, W, Us, wrow, qscale, qzero);
      const float wj = ws[JJ];
      const float sc = st.scale;
      const float q = sc > 0.f ? fminf(fmaxf(code_of(wj, sc, st.rscale), st.cmin), st.cmax) : 0.f;
      const float err = (wj - q * sc) * inv_u[j];
      code_row[j] = static_cast<int8_t>(q);
      e[JJ] = err;
      const float4* urow = reinterpret_cast<const float4*>(Us + j * B + c0);
#pragma unroll
      for (int k4 = (JJ + 1) >> 2; k4 < SUB / 4; ++k4) {  // U is 0 on and below the diagonal
        const float4 u = urow[k4];
        ws[4 * k4 + 0] = fmaf(-err, u.x, ws[4 * k4 + 0]);
        ws[4 * k4 + 1] = fmaf(-err, u.y, ws[4 * k4 + 1]);
        ws[4 * k4 + 2] = fmaf(-err, u.z, ws[4 * k4 + 2]);
        ws[4 * k4 + 3] = fmaf(-err, u.w, ws[4 * k4 + 3]);
      }
    } else {
      e[JJ] = 0.f;
    }
    sweep_col<GENERAL, JJ + 1>(ws, e, c0, st, W, Us, inv_u, wrow, code_row, qscale, qzero);
  }
}

// GENERAL = false: every group start of the block falls on a 32-column window
// boundary (g a multiple of 32), so scales are taken once per window, outside
// the unrolled column chain; GENERAL = true handles any g.
template <bool GENERAL>
__global__ void __launch_bounds__(R, 1)
    sweep_block_kernel(float* __restrict__ W, int64_t out, int64_t in,
                       const float* __restrict__ U, int64_t b, int kb, int bits, int g,
                       int8_t* __restrict__ codes, float* __restrict__ qscale,
                       uint8_t* __restrict__ qzero, float* __restrict__ Err, DeviceStatus* st) {
  extern __shared__ __align__(16) float smem[];
  float* Us = smem;                     // [B][B], strictly upper part of U[b:e, b:e]
  float* inv_u = Us + B * B;            // [B], 1 / U[j][j]
  float* Wr = inv_u + B;                // [R][LDW], row state; errors replace used columns
  int8_t* Cs = reinterpret_cast<int8_t*>(Wr + R * LDW);  // [R][LDC]
  pdl_launch_dependents();
  pdl_wait();  // W and U come from the previous kernels
  if (status_bad(st)) return;
  const int tid = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * R;

  // Tiles arrive by asynchronous copies (16-byte when the block start allows);
  // a second pass zeroes what the column loop must see as zero.
  const int rows_here = static_cast<int>(std::min<int64_t>(R, out - row0));
  if ((b & 3) == 0) {
    const int kq = (kb + 3) >> 2;  // b + 4*kq <= in since in % 8 == 0
    for (int idx = tid; idx < kb * kq; idx += R) {
      const int r = idx / kq, c = (idx - r * kq) * 4;
      cp_async16(Us + r * B + c, U + (b + r) * in + b + c);
    }
    for (int idx = tid; idx < rows_here * kq; idx += R) {
      const int r = idx / kq, c = (idx - r * kq) * 4;
      cp_async16(Wr + r * LDW + c, W + (row0 + r) * in + b + c);
    }
  } else {
    for (int idx = tid; idx < kb * kb; idx += R) {
      const int r = idx / kb, c = idx - r * kb;
      cp_async4(Us + r * B + c, U + (b + r) * in + b + c);
    }
    for (int idx = tid; idx < rows_here * kb; idx += R) {
      const int r = idx / kb, c = idx - r * kb;
      cp_async4(Wr + r * LDW + c, W + (row0 + r) * in + b + c);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  for (int idx = tid; idx < B * B; idx += R) {
    const int r = idx >> 7, c = idx & (B - 1);
    if (r >= kb || c >= kb || c <= r) Us[idx] = 0.f;
  }
  for (int idx = tid; idx < R * B; idx += R) {
    const int r = idx >> 7, c = idx & (B - 1);
    if (r >= rows_here || c >= kb) Wr[r * LDW + c] = 0.f;
  }
  for (int j = tid; j < B; j += R) inv_u[j] = (j < kb) ? 1.f / U[(b + j) * in + b + j] : 0.f;
  __syncthreads();

  SweepRow rs;
  const int qmax = (1 << (bits - 1)) - 1;
  rs.fqmax = qzero ? static_cast<float>((1 << bits) - 1) : static_cast<float>(qmax);
  rs.cmin = static_cast<float>(-qmax - 1);
  rs.cmax = static_cast<float>(qmax);
  rs.kb = kb;
  rs.b = b;
  rs.in = in;
  rs.g = g;
  rs.ngroups = (in + g - 1) / g;
  rs.row = row0 + tid;
  rs.valid = rs.row < out;
  const int64_t boff = b % g;
  // a group that started in an earlier block keeps its scale (and zero-point)
  rs.scale = (boff != 0 && rs.valid) ? qscale[rs.row * rs.ngroups + b / g] : 0.f;
  rs.rscale = rs.scale > 0.f ? __frcp_rn(rs.scale) : 0.f;
  if (qzero && boff != 0) {
    const float z = rs.valid ? static_cast<float>(qzero[rs.row * rs.ngroups + b / g]) : 0.f;
    rs.cmin = -z;
    rs.cmax = rs.fqmax - z;
  }
  rs.next_gs = (boff == 0) ? 0 : g - boff;

  float* wrow = Wr + tid * LDW;
  int8_t* crow = Cs + tid * LDC;
  for (int c0 = 0; c0 < kb; c0 += SUB) {
    float ws[SUB], e[SUB];
#pragma unroll
    for (int k4 = 0; k4 < SUB / 4; ++k4) {
      const float4 v = reinterpret_cast<const float4*>(wrow + c0)[k4];
      ws[4 * k4] = v.x;
      ws[4 * k4 + 1] = v.y;
      ws[4 * k4 + 2] = v.z;
      ws[4 * k4 + 3] = v.w;
    }
    if (!GENERAL && c0 == rs.next_gs) {
#pragma unroll
      for (int p = 0; p < SUB; ++p) e[p] = 0.f;
      group_start(ws, e, 0, c0, rs, W, Us, wrow, qscale, qzero);
    }
    sweep_col<GENERAL, 0>(ws, e, c0, rs, W, Us, inv_u, wrow, crow, qscale, qzero);
#pragma unroll
    for (int k4 = 0; k4 < SUB / 4; ++k4)
      reinterpret_cast<float4*>(wrow + c0)[k4] =
          make_float4(e[4 * k4], e[4 * k4 + 1], e[4 * k4 + 2], e[4 * k4 + 3]);
    // the window's errors update every later column of the block
    for (int k4 = (c0 + SUB) / 4; k4 < B / 4; ++k4) {
      float4 acc = reinterpret_cast<const float4*>(wrow)[k4];
#pragma unroll
      for (int p = 0; p < SUB; ++p) {
        const float4 u = reinterpret_cast<const float4*>(Us + (c0 + p) * B)[k4];
        acc.x = fmaf(-e[p], u.x, acc.x);
        acc.y = fmaf(-e[p], u.y, acc.y);
        acc.z = fmaf(-e[p], u.z, acc.z);
        acc.w = fmaf(-e[p], u.w, acc.w);
      }
      reinterpret_cast<float4*>(wrow)[k4] = acc;
    }
  }

  __syncthreads();
  for (int idx = tid; idx < R * B; idx += R) {  // coalesced write-out
    const int r = idx / B, c = idx % B;
    if (row0 + r < out && c < kb) {
      codes[(row0 + r) * in + b + c] = Cs[r * LDC + c];
      Err[(row0 + r) * B + c] = Wr[r * LDW + c];
    }
  }
}

// Blocks that hold no group start other than (possibly) their first column,
// which is every block when g % 128 == 0.  16 warps: warp w owns rows
// 32 (w % 4) .. + 31 (one per lane) and window q = w / 4 (block columns 32q ..
// 32q + 31) in registers.  Phase p (0..3): the quarter-p warps apply the errors
// of window p - 1 to their window and run its serial column loop; the warps of
// later windows apply the same errors at the same time.  Window errors replace
// the used columns of the row state in shared memory.
constexpr int QT = 4 * R;  // threads of the quartered kernel

__global__ void __launch_bounds__(QT, 1)
    sweep_quarters_kernel(float* __restrict__ W, int64_t out, int64_t in,
                          const float* __restrict__ U, int64_t b, int kb, int bits, int g,
                          int8_t* __restrict__ codes, float* __restrict__ qscale,
                          uint8_t* __restrict__ qzero, float* __restrict__ Err,
                          DeviceStatus* st) {
  extern __shared__ __align__(16) float smem[];
  float* Us = smem;                     // [B][B], strictly upper part of U[b:e, b:e]
  float* inv_u = Us + B * B;            // [B], 1 / U[j][j]
  float* Wr = inv_u + B;                // [R][LDW], row state; errors replace used columns
  int8_t* Cs = reinterpret_cast<int8_t*>(Wr + R * LDW);  // [R][LDC]
  float* scale_s = reinterpret_cast<float*>(Cs + R * LDC);  // [R]
  float* zero_s = scale_s + R;                              // [R] (asymmetric groups)
  pdl_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // window q's four warps sit on the four schedulers (warp w issues from w % 4)
  const int q = warp >> 2;                   // window
  const int lrow = (warp & 3) * 32 + lane;   // row within the CTA
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * R;
  const int rows_here = static_cast<int>(std::min<int64_t>(R, out - row0));
  const bool vec = (b & 3) == 0;  // 16-byte aligned rows at column b (in % 4 == 0 too)

  // U is read before the wait: no kernel that lets its successor start early
  // (the GEMMs, the factor, the sweep) writes U, so it is complete once this
  // kernel runs.  The part on and below the diagonal (and past kb) is zeroed in
  // the same pass.
  if (vec) {
    for (int idx = tid; idx < B * (B / 4); idx += QT) {
      const int r = idx / (B / 4), c = (idx - r * (B / 4)) * 4;
      float* dst = Us + r * B + c;
      if (r < kb && c > r && c + 3 < kb) {
        cp_async16(dst, U + (b + r) * in + b + c);
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (r < kb && c + t > r && c + t < kb)
            cp_async4(dst + t, U + (b + r) * in + b + c + t);
          else
            dst[t] = 0.f;
        }
      }
    }
  } else {
    for (int idx = tid; idx < B * B; idx += QT) {
      const int r = idx / B, c = idx - r * B;
      if (r < kb && c > r && c < kb)
        cp_async4(Us + idx, U + (b + r) * in + b + c);
      else
        Us[idx] = 0.f;
    }
  }
  for (int j = tid; j < B; j += QT) inv_u[j] = (j < kb) ? 1.f / U[(b + j) * in + b + j] : 0.f;
  pdl_wait();  // W comes from the previous kernels
  if (status_bad(st)) {
    cp_async_wait_all();
    return;
  }
  if (vec) {
    const int kq = (kb + 3) >> 2;
    for (int idx = tid; idx < R * (B / 4); idx += QT) {
      const int r = idx / (B / 4), c4 = idx - r * (B / 4);
      float* dst = Wr + r * LDW + 4 * c4;
      if (r < rows_here && c4 < kq)
        cp_async16(dst, W + (row0 + r) * in + b + 4 * c4);  // kb % 4 == 0 or zero-padded below
      else
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else {
    for (int idx = tid; idx < R * B; idx += QT) {
      const int r = idx / B, c = idx - r * B;
      if (r < rows_here && c < kb)
        cp_async4(Wr + r * LDW + c, W + (row0 + r) * in + b + c);
      else
        Wr[r * LDW + c] = 0.f;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (vec && (kb & 3) != 0) {  // the last 16-byte chunk of a ragged block read past kb
    for (int idx = tid; idx < R * 4; idx += QT) {
      const int r = idx >> 2, c = (kb & ~3) + (idx & 3);
      if (c >= kb) Wr[r * LDW + c] = 0.f;
    }
    __syncthreads();
  }

  SweepRow rs;
  const int qmax = (1 << (bits - 1)) - 1;
  rs.fqmax = qzero ? static_cast<float>((1 << bits) - 1) : static_cast<float>(qmax);
  rs.cmin = static_cast<float>(-qmax - 1);
  rs.cmax = static_cast<float>(qmax);
  rs.kb = kb;
  rs.b = b;
  rs.in = in;
  rs.g = g;
  rs.ngroups = (in + g - 1) / g;
  rs.row = row0 + lrow;
  rs.valid = rs.row < out;
  rs.next_gs = INT64_MAX;  // no group start inside the window loops
  float* wrow = Wr + lrow * LDW;
  int8_t* crow = Cs + lrow * LDC;
  if (q == 0) {
    // the row's scale: a group starts here (from the current weights of
    // [b, b + g), past the block read from W), or it continues from earlier
    float sc, z = 0.f;
    if (b % g == 0) {
      const int64_t gend = std::min<int64_t>(b + g, in);
      float m = 0.f;
      if (qzero == nullptr) {
        for (int c4 = 0; c4 < B / 4; ++c4) {  // columns past kb are zero
          const float4 v = reinterpret_cast<const float4*>(wrow)[c4];
          m = fmaxf(fmaxf(m, fmaxf(fabsf(v.x), fabsf(v.y))), fmaxf(fabsf(v.z), fabsf(v.w)));
        }
        if (rs.valid)
          for (int64_t c = b + kb; c < gend; ++c) m = fmaxf(m, fabsf(W[rs.row * in + c]));
        sc = __fdiv_rn(m, rs.fqmax);
      } else {
        // max(0, max w) and min(0, min w); zero columns past kb change neither
        float mn = 0.f;
        for (int c4 = 0; c4 < B / 4; ++c4) {
          const float4 v = reinterpret_cast<const float4*>(wrow)[c4];
          m = fmaxf(fmaxf(m, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
          mn = fminf(fminf(mn, fminf(v.x, v.y)), fminf(v.z, v.w));
        }
        if (rs.valid)
          for (int64_t c = b + kb; c < gend; ++c) {
            m = fmaxf(m, W[rs.row * in + c]);
            mn = fminf(mn, W[rs.row * in + c]);
          }
        asym_params(m, mn, rs, qzero, b / g);
        sc = rs.scale;
        z = -rs.cmin;
      }
      if (rs.valid) qscale[rs.row * rs.ngroups + b / g] = sc;
    } else {
      sc = rs.valid ? qscale[rs.row * rs.ngroups + b / g] : 0.f;
      if (qzero && rs.valid) z = static_cast<float>(qzero[rs.row * rs.ngroups + b / g]);
    }
    scale_s[lrow] = sc;
    zero_s[lrow] = z;
  }
  const int c0 = SUB * q;
  // ws holds the window's weights; a used column's slot then holds its error
  // (U is zero on and below the diagonal, so later updates leave it unchanged)
  float ws[SUB];
#pragma unroll
  for (int k4 = 0; k4 < SUB / 4; ++k4) {
    const float4 v = reinterpret_cast<const float4*>(wrow + c0)[k4];
    ws[4 * k4] = v.x;
    ws[4 * k4 + 1] = v.y;
    ws[4 * k4 + 2] = v.z;
    ws[4 * k4 + 3] = v.w;
  }
  __syncthreads();
  rs.scale = scale_s[lrow];
  rs.rscale = rs.scale > 0.f ? __frcp_rn(rs.scale) : 0.f;
  if (qzero) {
    rs.cmin = -zero_s[lrow];
    rs.cmax = rs.fqmax - zero_s[lrow];
  }

  for (int p = 0; p < 4; ++p) {
    if (q >= p && SUB * p < kb) {
      if (p > 0) {
        // errors of window p - 1 onto this window
        const int cp = SUB * (p - 1);
#pragma unroll 1
        for (int i4 = 0; i4 < SUB / 4; ++i4) {
          const float4 e4 = reinterpret_cast<const float4*>(wrow + cp)[i4];
          const float ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float4* urow = reinterpret_cast<const float4*>(Us + (cp + 4 * i4 + t) * B + c0);
#pragma unroll
            for (int k4 = 0; k4 < SUB / 4; ++k4) {
              const float4 u = urow[k4];
              ws[4 * k4 + 0] = fmaf(-ev[t], u.x, ws[4 * k4 + 0]);
              ws[4 * k4 + 1] = fmaf(-ev[t], u.y, ws[4 * k4 + 1]);
              ws[4 * k4 + 2] = fmaf(-ev[t], u.z, ws[4 * k4 + 2]);
              ws[4 * k4 + 3] = fmaf(-ev[t], u.w, ws[4 * k4 + 3]);
            }
          }
        }
      }
      if (q == p) {
        sweep_col<false, 0>(ws, ws, c0, rs, W, Us, inv_u, wrow, crow, qscale, qzero);
#pragma unroll
        for (int k4 = 0; k4 < SUB / 4; ++k4)
          reinterpret_cast<float4*>(wrow + c0)[k4] =
              make_float4(ws[4 * k4], ws[4 * k4 + 1], ws[4 * k4 + 2], ws[4 * k4 + 3]);
      }
    }
    __syncthreads();
  }

  // coalesced write-out: error rows as float4 (Err rows are 128 floats; the row
  // state stride LDW = 132 floats keeps 16-byte alignment), codes 4 at a time
  for (int idx = tid; idx < R * (B / 4); idx += QT) {
    const int r = idx / (B / 4), c4 = idx - r * (B / 4);
    if (r < rows_here && 4 * c4 < kb)
      reinterpret_cast<float4*>(Err + (row0 + r) * B)[c4] =
          reinterpret_cast<const float4*>(Wr + r * LDW)[c4];
  }
  // 4 codes per access: the staging rows (LDC = 132 bytes) are 4-byte aligned
  const bool cvec = (b & 3) == 0 && (in & 3) == 0 && (kb & 3) == 0;
  if (cvec) {
    for (int idx = tid; idx < R * (B / 4); idx += QT) {
      const int r = idx / (B / 4), c4 = idx - r * (B / 4);
      if (r < rows_here && 4 * c4 < kb)
        *reinterpret_cast<uint32_t*>(codes + (row0 + r) * in + b + 4 * c4) =
            *reinterpret_cast<const uint32_t*>(Cs + r * LDC + 4 * c4);
    }
  } else {
    for (int idx = tid; idx < R * B; idx += QT) {
      const int r = idx / B, c = idx % B;
      if (r < rows_here && c < kb) codes[(row0 + r) * in + b + c] = Cs[r * LDC + c];
    }
  }
}

}  // namespace

// Column blocks of width <= 128 where each group start inside a block has its
// whole group inside that block.
static void block_partition(int64_t in, int g, std::vector<std::pair<int64_t, int64_t>>* blocks) {
  blocks->clear();
  int64_t b = 0;
  while (b < in) {
    int64_t e = std::min<int64_t>(b + B, in);
    for (int64_t s = (b / g + 1) * g; s < e; s += g) {
      if (std::min<int64_t>(s + g, in) > e) {
        e = s;
        break;
      }
    }
    blocks->push_back({b, e});
    b = e;
  }
}

int run_gptq_sweep(float* Wq, int64_t out, int64_t in, const float* U, int bits, int g,
                   int8_t* codes, float* qscale, uint8_t* qzero, float* Err, DeviceStatus* st,
                   cudaStream_t stream) {
  static bool attr_set[64] = {};
  static bool quarters_attr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(sweep_block_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSweepSmem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(sweep_block_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSweepSmem) !=
            cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  // with g % 128 == 0 no block holds a group start past its first column
  const bool quartered = g % B == 0;
  if (quartered && dev < 64 && !quarters_attr[dev]) {
    if (cudaFuncSetAttribute(sweep_quarters_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kQuartersSmem) != cudaSuccess)
      return PIQ_ERR_CUDA;
    quarters_attr[dev] = true;
  }
  std::vector<std::pair<int64_t, int64_t>> blocks;
  block_partition(in, g, &blocks);
  const unsigned grid = static_cast<unsigned>(ceil_div(out, R));
  for (const auto& be : blocks) {
    const int64_t b = be.first, e = be.second;
    const int kb = static_cast<int>(e - b);
    // do all group starts inside the block fall on window boundaries?
    bool aligned = true;
    for (int64_t gs = (b % g == 0) ? b : (b / g + 1) * g; gs < e; gs += g)
      aligned = aligned && ((gs - b) % SUB == 0);
    note_launch();
    const cudaError_t le =
        quartered ? launch_pdl(sweep_quarters_kernel, dim3(grid), dim3(QT), kQuartersSmem, stream,
                               Wq, out, in, U, b, kb, bits, g, codes, qscale, qzero, Err, st)
        : aligned ? launch_pdl(sweep_block_kernel<false>, dim3(grid), dim3(R), kSweepSmem, stream, Wq,
                             out, in, U, b, kb, bits, g, codes, qscale, qzero, Err, st)
                : launch_pdl(sweep_block_kernel<true>, dim3(grid), dim3(R), kSweepSmem, stream, Wq,
                             out, in, U, b, kb, bits, g, codes, qscale, qzero, Err, st);
    if (le != cudaSuccess) return PIQ_ERR_CUDA;
    if (e < in) {
      // W[:, e:] -= Err[:, :kb] U[b:e, e:]
      int rc = launch_gemm_f32(static_cast<int>(out), static_cast<int>(in - e), kb, -1.f, Err, B,
                                U + b * in + e, in, false, 1.f, Wq + e, in, 0, st, stream);
      if (rc != PIQ_OK) return rc;
    }
  }
  return PIQ_OK;
}

}  // namespace piq
