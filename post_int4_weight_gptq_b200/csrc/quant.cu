// Bandwidth-bound kernels of the quantization path.
//
//   colstats      per input channel: sum |x| (AWQ's mean|x_j|, "GPTQ versus AWQ
//                 objectives", AWQ paragraph of "A strong answer") and sum x^2
//                 (= diag(X^T X), the act-order key of "What interviewers probe
//                 next"), one pass over X, FP64 accumulation.
//   awq_delta     for every alpha of the grid: s = mean|x|^alpha, W' = W diag(s),
//                 symmetric group round-to-nearest of W', and
//                 D = W - code * scale / s stored as bf16 for the error GEMM.
//   group_quant   codes + fp32 scales of W diag(s) for one s (AWQ's chosen alpha;
//                 s = 1 gives plain group RTN, the toy table's first column).
//   pack          codes -> uint32 nibbles, fp32 -> fp16 scales, act-order
//                 column un-permutation and g_idx, and D = W - code * fp16(scale)
//                 (bf16) for the output-error GEMM, in one pass.
//   scale_upper   H' = diag(1/s) H diag(1/s) in place, the proxy Hessian of the
//                 AWQ-scaled inputs X diag(1/s) (AWQ's scaling first, GPTQ's
//                 rounding after: the serving decision list of "GPTQ versus AWQ
//                 objectives"); also checks s.
#include <algorithm>

#include "internal.h"

namespace piq {

namespace {

// ------------------------------------------------------------------- colstats
// grid (ceil(in/256), splits); 8 warps; lane owns 8 consecutive columns.
// SQ = 0: sum |x| per column, two rows added in FP32 (round to nearest) before
// each FP64 addition (relative error below 2^-24 of the sum, for the AWQ
// channel means); SQ = 1: sum x^2 per column, every square (exact in FP32 for
// bf16 inputs) added in FP64, so the act-order ranking sees exact sums.
template <int SQ>
__global__ void __launch_bounds__(256) colstats_kernel(const uint16_t* __restrict__ X, int64_t n,
                                                       int64_t in, int splits,
                                                       double* __restrict__ part) {
  __shared__ double sh[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t col = static_cast<int64_t>(blockIdx.x) * 256 + lane * 8;
  const int64_t rows_per = (n + splits - 1) / splits;
  const int64_t r0 = blockIdx.y * rows_per;
  const int64_t r1 = std::min<int64_t>(n, r0 + rows_per);
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  auto term = [](uint16_t b) {
    const float x = bf16_bits_to_float(b);
    return SQ ? x * x : fabsf(x);
  };
  // one row: every term to FP64
  auto add1 = [&](const uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += static_cast<double>(term(static_cast<uint16_t>(w[i] & 0xFFFFu)));
      acc[2 * i + 1] += static_cast<double>(term(static_cast<uint16_t>(w[i] >> 16)));
    }
  };
  // two rows: |x| terms summed in FP32 first (SQ = 0 only)
  auto add2 = [&](const uint4 va, const uint4 vb) {
    const uint32_t a[4] = {va.x, va.y, va.z, va.w}, b[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += static_cast<double>(__fadd_rn(term(static_cast<uint16_t>(a[i] & 0xFFFFu)),
                                                  term(static_cast<uint16_t>(b[i] & 0xFFFFu))));
      acc[2 * i + 1] += static_cast<double>(
          __fadd_rn(term(static_cast<uint16_t>(a[i] >> 16)), term(static_cast<uint16_t>(b[i] >> 16))));
    }
  };
  if (col < in) {
    // four rows in flight per thread; rows are added in the same order either way
    int64_t r = r0 + warp;
    for (; r + 24 < r1; r += 32) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(X + r * in + col));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(X + (r + 8) * in + col));
      const uint4 v2 = __ldg(reinterpret_cast<const uint4*>(X + (r + 16) * in + col));
      const uint4 v3 = __ldg(reinterpret_cast<const uint4*>(X + (r + 24) * in + col));
      if (SQ) {
        add1(v0);
        add1(v1);
        add1(v2);
        add1(v3);
      } else {
        add2(v0, v1);
        add2(v2, v3);
      }
    }
    for (; r < r1; r += 8) add1(__ldg(reinterpret_cast<const uint4*>(X + r * in + col)));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) sh[warp][lane * 8 + i] = acc[i];
  __syncthreads();
  const int c = threadIdx.x;
  const int64_t gc = static_cast<int64_t>(blockIdx.x) * 256 + c;
  if (gc < in) {
    double a = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) a += sh[w][c];
    part[static_cast<int64_t>(blockIdx.y) * in + gc] = a;
  }
}

__global__ void colstats_finish_kernel(const double* __restrict__ part, int64_t n, int64_t in,
                                       int splits, int mean, double* out) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= in) return;
  double a = 0.0;
  for (int s = 0; s < splits; ++s) a += part[static_cast<int64_t>(s) * in + c];
  out[c] = mean ? a / static_cast<double>(n) : a;
}

// --------------------------------------------------------------------- gather
// Wq[r][p] = W[r][perm[p]] * cs[perm[p]] (perm == NULL: identity; cs == NULL:
// no scaling), four positions per thread (in % 4 == 0 and 16-byte aligned
// rows, perm and cs; the launcher checks).  The product is the same fp32
// multiply pack_kernel makes, so both see the same W diag(s).
__global__ void gather_columns_kernel(const float* __restrict__ W, int64_t out, int64_t in,
                                      const int32_t* __restrict__ perm,
                                      const float* __restrict__ cs, float* __restrict__ Wq) {
  const int64_t total4 = out * in / 4;
  const int64_t in4 = in / 4;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total4;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 v;
    const int64_t r = idx / in4, p = (idx - r * in4) * 4;
    int4 c = make_int4(static_cast<int>(p), static_cast<int>(p + 1), static_cast<int>(p + 2),
                       static_cast<int>(p + 3));
    if (perm == nullptr) {
      v = __ldg(reinterpret_cast<const float4*>(W) + idx);
    } else {
      c = __ldg(reinterpret_cast<const int4*>(perm + p));
      const float* wr = W + r * in;
      v = make_float4(__ldg(wr + c.x), __ldg(wr + c.y), __ldg(wr + c.z), __ldg(wr + c.w));
    }
    if (cs != nullptr) {
      if (perm == nullptr) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(cs + p));
        v = make_float4(v.x * t.x, v.y * t.y, v.z * t.z, v.w * t.w);
      } else {
        v = make_float4(v.x * __ldg(cs + c.x), v.y * __ldg(cs + c.y), v.z * __ldg(cs + c.z),
                        v.w * __ldg(cs + c.w));
      }
    }
    reinterpret_cast<float4*>(Wq)[idx] = v;
  }
}

// -------------------------------------------------------------- scale_upper
// H[k][j] /= s_k s_j for the 4-column chunks that hold j >= k (the valid upper
// triangle; the rest is never read), one rounding from FP64.  A block with
// blockIdx.x == 0 checks s_k (finite, > 0) for each of its rows.
__global__ void scale_upper_kernel(float* __restrict__ H, int64_t in, const float* __restrict__ s,
                                   DeviceStatus* st) {
  const int64_t in4 = in >> 2;
  for (int64_t k = blockIdx.y; k < in; k += gridDim.y) {
    const float sk = s[k];
    if (blockIdx.x == 0 && threadIdx.x == 0 && !(sk > 0.f && sk <= 3.4028235e38f))
      set_status(st, PIQ_ERR_INVALID_ARG, static_cast<int>(k));
    const double rk = 1.0 / static_cast<double>(sk);
    float4* row = reinterpret_cast<float4*>(H + k * in);
    const float4* s4 = reinterpret_cast<const float4*>(s);
    for (int64_t t = (k >> 2) + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         t < in4; t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const float4 h = row[t];
      const float4 sj = __ldg(s4 + t);
      row[t] = make_float4(static_cast<float>(static_cast<double>(h.x) * rk / sj.x),
                           static_cast<float>(static_cast<double>(h.y) * rk / sj.y),
                           static_cast<float>(static_cast<double>(h.z) * rk / sj.z),
                           static_cast<float>(static_cast<double>(h.w) * rk / sj.w));
    }
  }
}

// The same on an fp64 H (the upper triangle, rows from their diagonal on).
__global__ void scale_upper64_kernel(double* __restrict__ H, int64_t in,
                                     const float* __restrict__ s, DeviceStatus* st) {
  for (int64_t k = blockIdx.y; k < in; k += gridDim.y) {
    const float sk = s[k];
    if (blockIdx.x == 0 && threadIdx.x == 0 && !(sk > 0.f && sk <= 3.4028235e38f))
      set_status(st, PIQ_ERR_INVALID_ARG, static_cast<int>(k));
    const double rk = 1.0 / static_cast<double>(sk);
    double* row = H + k * in;
    for (int64_t j = k + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < in;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
      row[j] = row[j] * rk / static_cast<double>(__ldg(s + j));
  }
}

// sumsq[j] /= s_j^2 in FP64 (s_j^2 is exact there): diag of the scaled Hessian,
// the act-order key of the scaled layer.
__global__ void scale_sumsq_kernel(double* __restrict__ sumsq, int64_t in,
                                   const float* __restrict__ s) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < in) {
    const double sj = static_cast<double>(s[j]);
    sumsq[j] = sumsq[j] / (sj * sj);
  }
}

// ----------------------------------------------------------------------- pack
// One thread per uint32 word (8 memory-order columns).  With cs, the delta is
// taken against W0[r][c] * cs[c] (the scaled layer the codes belong to).
__global__ void pack_kernel(const int8_t* __restrict__ codes, const float* __restrict__ qscale,
                            const uint8_t* __restrict__ qzero,
                            const int32_t* __restrict__ invperm, int64_t out, int64_t in,
                            int bits, int g, const float* __restrict__ W0,
                            const float* __restrict__ cs, uint32_t* __restrict__ qweight,
                            uint16_t* __restrict__ scales16, uint16_t* __restrict__ dW,
                            float* __restrict__ dW32, int32_t* __restrict__ g_idx) {
  const int64_t words = in / 8;
  const int64_t ngroups = (in + g - 1) / g;
  const int64_t total = out * words;
  const int off = 1 << (bits - 1);
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / words, wd = idx - r * words;
    const int8_t* crow = codes + r * in;
    const float* srow = qscale + r * ngroups;
    uint32_t word = 0;
    float d32[8];
    float w0[8];
    const bool delta = dW != nullptr || dW32 != nullptr;
    if (delta) {
      const float4 a = *reinterpret_cast<const float4*>(W0 + r * in + wd * 8);
      const float4 b = *reinterpret_cast<const float4*>(W0 + r * in + wd * 8 + 4);
      w0[0] = a.x; w0[1] = a.y; w0[2] = a.z; w0[3] = a.w;
      w0[4] = b.x; w0[5] = b.y; w0[6] = b.z; w0[7] = b.w;
      if (cs != nullptr) {
        const float4 sa = __ldg(reinterpret_cast<const float4*>(cs + wd * 8));
        const float4 sb = __ldg(reinterpret_cast<const float4*>(cs + wd * 8 + 4));
        w0[0] *= sa.x; w0[1] *= sa.y; w0[2] *= sa.z; w0[3] *= sa.w;
        w0[4] *= sb.x; w0[5] *= sb.y; w0[6] *= sb.z; w0[7] *= sb.w;
      }
    }
    if (invperm == nullptr && (g & 7) == 0) {
      // natural order, the word inside one group: one 8-byte load of the codes,
      // one scale (and zero-point) for the word
      const uint2 cw = *reinterpret_cast<const uint2*>(crow + wd * 8);
      const int64_t grp = (wd * 8) / g;
      const int zp = qzero ? static_cast<int>(qzero[r * ngroups + grp]) : off;
      const float s16 = delta ? __half2float(__float2half_rn(srow[grp])) : 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int code = static_cast<int8_t>(((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xFFu);
        word |= static_cast<uint32_t>(code + zp) << (4 * k);
        if (delta) d32[k] = w0[k] - static_cast<float>(code) * s16;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t c = wd * 8 + k;
        const int64_t p = invperm ? invperm[c] : c;
        const int code = crow[p];
        const int zp = qzero ? static_cast<int>(qzero[r * ngroups + p / g]) : off;
        word |= static_cast<uint32_t>(code + zp) << (4 * k);
        if (delta) {
          const float s16 = __half2float(__float2half_rn(srow[p / g]));
          d32[k] = w0[k] - static_cast<float>(code) * s16;
        }
      }
    }
    qweight[idx] = word;
    if (dW32) {
      float4* dst = reinterpret_cast<float4*>(dW32 + r * in + wd * 8);
      dst[0] = make_float4(d32[0], d32[1], d32[2], d32[3]);
      dst[1] = make_float4(d32[4], d32[5], d32[6], d32[7]);
    }
    if (dW) {
      uint4 o;
      o.x = floats_to_bf16x2_bits(d32[0], d32[1]);
      o.y = floats_to_bf16x2_bits(d32[2], d32[3]);
      o.z = floats_to_bf16x2_bits(d32[4], d32[5]);
      o.w = floats_to_bf16x2_bits(d32[6], d32[7]);
      *reinterpret_cast<uint4*>(dW + r * in + wd * 8) = o;
    }
  }
  // fp16 scales and the group index
  const int64_t ns = out * ngroups;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < ns;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x)
    scales16[idx] = __half_as_ushort(__float2half_rn(qscale[idx]));
  if (g_idx) {
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < in;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x)
      g_idx[c] = static_cast<int32_t>((invperm ? invperm[c] : c) / g);
  }
}

// ------------------------------------------------------------------------ AWQ
__global__ void awq_scale_table_kernel(const double* __restrict__ mean_abs, int64_t in,
                                       const float* __restrict__ alphas, int n_alpha,
                                       float* __restrict__ s_table) {
  const int64_t total = static_cast<int64_t>(n_alpha) * in;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int a = static_cast<int>(idx / in);
    const double m = mean_abs[idx - a * in];
    const float sv = m > 0.0 ? static_cast<float>(pow(m, static_cast<double>(alphas[a]))) : 1.f;
    s_table[idx] = sv;
    s_table[total + idx] = 1.f / sv;  // reciprocals follow the scales
  }
}

// Group scale and codes of W diag(s) for one (row, group): one warp.
struct GroupQ {
  float scale;
};

__device__ __forceinline__ float group_scale(const float* wrow, const float* s, int64_t c0,
                                             int64_t c1, float fqmax, int lane) {
  float m = 0.f;
  for (int64_t c = c0 + lane; c < c1; c += 32) {
    const float v = s ? wrow[c] * s[c] : wrow[c];
    m = fmaxf(m, fabsf(v));
  }
  return __fdiv_rn(warp_max(m), fqmax);
}

__device__ __forceinline__ float quant_code(float v, float scale, float cmin, float cmax) {
  return scale > 0.f ? fminf(fmaxf(rintf(__fdiv_rn(v, scale)), cmin), cmax) : 0.f;
}

// D_a[r][c] = W - code * scale / s for every alpha a; one warp per (row, group).
__global__ void awq_delta_kernel(const float* __restrict__ W, int64_t out, int64_t in, int bits,
                                 int g, const float* __restrict__ s_table, int n_alpha,
                                 uint16_t* __restrict__ dW) {
  const int64_t ngroups = (in + g - 1) / g;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int qmax = (1 << (bits - 1)) - 1;
  const float fqmax = static_cast<float>(qmax), cmin = static_cast<float>(-qmax - 1),
              cmax = static_cast<float>(qmax);
  for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wi < out * ngroups; wi += nwarps) {
    const int64_t r = wi / ngroups, grp = wi - r * ngroups;
    const int64_t c0 = grp * g, c1 = std::min<int64_t>(in, c0 + g);
    const float* wrow = W + r * in;
    for (int a = 0; a < n_alpha; ++a) {
      const float* s = s_table + static_cast<int64_t>(a) * in;
      const float scale = group_scale(wrow, s, c0, c1, fqmax, lane);
      uint16_t* drow = dW + (static_cast<int64_t>(a) * out + r) * in;
      for (int64_t c = c0 + lane; c < c1; c += 32) {
        const float w = wrow[c];
        const float q = quant_code(w * s[c], scale, cmin, cmax);
        drow[c] = float_to_bf16_bits(w - __fdiv_rn(q * scale, s[c]));
      }
    }
  }
}

// Vector form of awq_delta_kernel for g % 4 == 0 and g <= 128: lane l holds
// columns [4l, 4l+4) of one (row, group); W is read once for every alpha.  The
// code decision keeps the IEEE quotient W'/scale; the dequantised weight uses
// the precomputed reciprocal of s.
__global__ void __launch_bounds__(256)
    awq_delta_vec_kernel(const float* __restrict__ W, int64_t out, int64_t in, int bits, int g,
                         const float* __restrict__ s_table, int n_alpha,
                         uint16_t* __restrict__ dW) {
  const int64_t ngroups = (in + g - 1) / g;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int qmax = (1 << (bits - 1)) - 1;
  const float fqmax = static_cast<float>(qmax), cmin = static_cast<float>(-qmax - 1),
              cmax = static_cast<float>(qmax);
  const float* inv_table = s_table + static_cast<int64_t>(n_alpha) * in;
  for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wi < out * ngroups; wi += nwarps) {
    const int64_t r = wi / ngroups, grp = wi - r * ngroups;
    const int64_t c0 = grp * g;
    const int len = static_cast<int>(std::min<int64_t>(g, in - c0));  // multiple of 4
    const bool act = 4 * lane < len;
    const int64_t col = c0 + 4 * lane;
    const float4 w = act ? *reinterpret_cast<const float4*>(W + r * in + col)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int a = 0; a < n_alpha; ++a) {
      const int64_t off = static_cast<int64_t>(a) * in + col;
      const float4 sv = act ? *reinterpret_cast<const float4*>(s_table + off)
                            : make_float4(1.f, 1.f, 1.f, 1.f);
      const float4 iv = act ? *reinterpret_cast<const float4*>(inv_table + off)
                            : make_float4(1.f, 1.f, 1.f, 1.f);
      const float p0 = w.x * sv.x, p1 = w.y * sv.y, p2 = w.z * sv.z, p3 = w.w * sv.w;
      float m = fmaxf(fmaxf(fabsf(p0), fabsf(p1)), fmaxf(fabsf(p2), fabsf(p3)));
      const float scale = __fdiv_rn(warp_max(m), fqmax);
      const float q0 = quant_code(p0, scale, cmin, cmax), q1 = quant_code(p1, scale, cmin, cmax);
      const float q2 = quant_code(p2, scale, cmin, cmax), q3 = quant_code(p3, scale, cmin, cmax);
      if (act) {
        uint2 o;
        o.x = float_to_bf16_bits(w.x - q0 * scale * iv.x) |
              (static_cast<uint32_t>(float_to_bf16_bits(w.y - q1 * scale * iv.y)) << 16);
        o.y = float_to_bf16_bits(w.z - q2 * scale * iv.z) |
              (static_cast<uint32_t>(float_to_bf16_bits(w.w - q3 * scale * iv.w)) << 16);
        *reinterpret_cast<uint2*>(dW + (static_cast<int64_t>(a) * out + r) * in + col) = o;
      }
    }
  }
}

// The code rint(v / scale) clipped, from v * (1 / scale): the product differs
// from the IEEE quotient by at most two units in the last place, so it can only
// round differently within ~1e-6 of a half-integer; there the IEEE division
// decides.  Same result as quant_code.
__device__ __noinline__ float code_by_division(float v, float scale) {
  return rintf(__fdiv_rn(v, scale));
}

// D_a[r][c] = W - code * scale / s for every alpha a, for power-of-two g with
// 8 <= g <= 256 and in % 8 == 0.  Lane l of a warp holds columns 8l .. 8l+7 of a
// 256-column slice (g / 8 lanes per group) for kRows rows; per alpha the s and
// 1 / s of its columns are read once for all kRows rows.
constexpr int kRows = 4;
__global__ void __launch_bounds__(256, 3)
    awq_delta_rows_kernel(const float* __restrict__ W, int64_t out, int64_t in, int bits, int g,
                          const float* __restrict__ s_table, int n_alpha,
                          uint16_t* __restrict__ dW) {
  const int lane = threadIdx.x & 31;
  const int lg = g >> 3;  // lanes per group
  const int qmax = (1 << (bits - 1)) - 1;
  const float fqmax = static_cast<float>(qmax), cmin = static_cast<float>(-qmax - 1),
              cmax = static_cast<float>(qmax);
  const float* inv_table = s_table + static_cast<int64_t>(n_alpha) * in;
  const int64_t slices = (in + 255) / 256;
  const int64_t rblocks = (out + kRows - 1) / kRows;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wi < rblocks * slices; wi += nwarps) {
    const int64_t rb = wi / slices, sl = wi - rb * slices;
    const int64_t col = sl * 256 + 8 * lane;
    const bool act = col < in;  // in % 8 == 0: a lane is wholly in or out
    const int64_t r0 = rb * kRows;
    float w[kRows][8];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const bool ok = act && r0 + k < out;
      const float4 a = ok ? __ldg(reinterpret_cast<const float4*>(W + (r0 + k) * in + col))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 b = ok ? __ldg(reinterpret_cast<const float4*>(W + (r0 + k) * in + col + 4))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      w[k][0] = a.x; w[k][1] = a.y; w[k][2] = a.z; w[k][3] = a.w;
      w[k][4] = b.x; w[k][5] = b.y; w[k][6] = b.z; w[k][7] = b.w;
    }
    for (int al = 0; al < n_alpha; ++al) {
      float sv[8], iv[8];
      {
        const int64_t off = static_cast<int64_t>(al) * in + col;
        const float4 a = act ? __ldg(reinterpret_cast<const float4*>(s_table + off))
                             : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 b = act ? __ldg(reinterpret_cast<const float4*>(s_table + off + 4))
                             : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 c = act ? __ldg(reinterpret_cast<const float4*>(inv_table + off))
                             : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 d = act ? __ldg(reinterpret_cast<const float4*>(inv_table + off + 4))
                             : make_float4(1.f, 1.f, 1.f, 1.f);
        sv[0] = a.x; sv[1] = a.y; sv[2] = a.z; sv[3] = a.w;
        sv[4] = b.x; sv[5] = b.y; sv[6] = b.z; sv[7] = b.w;
        iv[0] = c.x; iv[1] = c.y; iv[2] = c.z; iv[3] = c.w;
        iv[4] = d.x; iv[5] = d.y; iv[6] = d.z; iv[7] = d.w;
      }
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        float p[8], m = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = w[k][e] * sv[e];
          m = fmaxf(m, fabsf(p[e]));
        }
        for (int o = 1; o < lg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float scale = __fdiv_rn(m, fqmax);
        const float rs = scale > 0.f ? __frcp_rn(scale) : 0.f;
        // rint(v / scale) from v * (1 / scale); within 1e-5 of a half-integer the
        // IEEE quotient decides (code_by_division), on one warp-uniform branch
        float q[8];
        bool near = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float t = p[e] * rs;
          q[e] = rintf(t);
          near |= fabsf(fabsf(t - q[e]) - 0.5f) < 1e-5f;
        }
        if (__any_sync(0xffffffffu, near)) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float t = p[e] * rs;
            if (fabsf(fabsf(t - rintf(t)) - 0.5f) < 1e-5f) q[e] = code_by_division(p[e], scale);
          }
        }
        uint16_t d16[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float qc = scale > 0.f ? fminf(fmaxf(q[e], cmin), cmax) : 0.f;
          d16[e] = float_to_bf16_bits(fmaf(-(qc * scale), iv[e], w[k][e]));
        }
        if (act && r0 + k < out) {
          uint4 o;
          o.x = d16[0] | (static_cast<uint32_t>(d16[1]) << 16);
          o.y = d16[2] | (static_cast<uint32_t>(d16[3]) << 16);
          o.z = d16[4] | (static_cast<uint32_t>(d16[5]) << 16);
          o.w = d16[6] | (static_cast<uint32_t>(d16[7]) << 16);
          *reinterpret_cast<uint4*>(dW + (static_cast<int64_t>(al) * out + r0 + k) * in + col) = o;
        }
      }
    }
  }
}

// codes + fp32 scales of W diag(s_table[sel]) (s_table == NULL: s = 1).
__global__ void group_quant_kernel(const float* __restrict__ W, int64_t out, int64_t in, int bits,
                                   int g, const float* __restrict__ s_table,
                                   const int* __restrict__ sel, int8_t* __restrict__ codes,
                                   float* __restrict__ qscale, float* __restrict__ s_out) {
  const int64_t ngroups = (in + g - 1) / g;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int qmax = (1 << (bits - 1)) - 1;
  const float fqmax = static_cast<float>(qmax), cmin = static_cast<float>(-qmax - 1),
              cmax = static_cast<float>(qmax);
  const float* s = s_table ? s_table + static_cast<int64_t>(sel ? *sel : 0) * in : nullptr;
  for (int64_t wi = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       wi < out * ngroups; wi += nwarps) {
    const int64_t r = wi / ngroups, grp = wi - r * ngroups;
    const int64_t c0 = grp * g, c1 = std::min<int64_t>(in, c0 + g);
    const float* wrow = W + r * in;
    const float scale = group_scale(wrow, s, c0, c1, fqmax, lane);
    if (lane == 0) qscale[r * ngroups + grp] = scale;
    for (int64_t c = c0 + lane; c < c1; c += 32) {
      const float v = s ? wrow[c] * s[c] : wrow[c];
      codes[r * in + c] = static_cast<int8_t>(quant_code(v, scale, cmin, cmax));
    }
  }
  if (s_out && s) {
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < in;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x)
      s_out[c] = s[c];
  }
}

__global__ void argmin_kernel(const double* err, int n, const float* alphas, int* best_idx,
                              float* best_alpha) {
  if (threadIdx.x != 0) return;
  int b = 0;
  for (int i = 1; i < n; ++i)
    if (err[i] < err[b]) b = i;
  *best_idx = b;
  if (best_alpha) *best_alpha = alphas[b];
}

// D = W - code * fp16(scale) / s, from the packed format (code = u - zero with
// zero-points, else u - 2^(bits-1)); one thread per word.
__global__ void dequant_delta_kernel(const float* __restrict__ W, int64_t out, int64_t in,
                                     const uint32_t* __restrict__ qweight,
                                     const uint16_t* __restrict__ scales16,
                                     const uint8_t* __restrict__ zeros,
                                     const int32_t* __restrict__ g_idx,
                                     const float* __restrict__ s, int bits, int g,
                                     uint16_t* __restrict__ dW, float* __restrict__ dW32,
                                     DeviceStatus* st) {
  const int64_t words = in / 8;
  const int64_t ngroups = (in + g - 1) / g;
  const int off = 1 << (bits - 1);
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < out * words; idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / words, wd = idx - r * words;
    const uint32_t word = qweight[idx];
    float d32[8];
    const float4 wa = __ldg(reinterpret_cast<const float4*>(W + r * in + wd * 8));
    const float4 wb = __ldg(reinterpret_cast<const float4*>(W + r * in + wd * 8 + 4));
    const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    int gi[8];
    if (g_idx && (reinterpret_cast<uintptr_t>(g_idx) & 15u) != 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) gi[k] = g_idx[wd * 8 + k];
    } else if (g_idx) {
      const int4 ga = __ldg(reinterpret_cast<const int4*>(g_idx + wd * 8));
      const int4 gb = __ldg(reinterpret_cast<const int4*>(g_idx + wd * 8 + 4));
      gi[0] = ga.x; gi[1] = ga.y; gi[2] = ga.z; gi[3] = ga.w;
      gi[4] = gb.x; gi[5] = gb.y; gi[6] = gb.z; gi[7] = gb.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) gi[k] = static_cast<int>((wd * 8 + k) / g);
    }
    float sv[8];
    if (s && (reinterpret_cast<uintptr_t>(s) & 15u) != 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) sv[k] = s[wd * 8 + k];
    } else if (s) {
      const float4 sa = __ldg(reinterpret_cast<const float4*>(s + wd * 8));
      const float4 sb = __ldg(reinterpret_cast<const float4*>(s + wd * 8 + 4));
      sv[0] = sa.x; sv[1] = sa.y; sv[2] = sa.z; sv[3] = sa.w;
      sv[4] = sb.x; sv[5] = sb.y; sv[6] = sb.z; sv[7] = sb.w;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t c = wd * 8 + k;
      int64_t grp = gi[k];
      if (grp < 0 || grp >= ngroups) {  // caller's group index out of range
        set_status(st, PIQ_ERR_INVALID_ARG, static_cast<int>(c));
        grp = 0;
      }
      const int zp = zeros ? static_cast<int>(zeros[r * ngroups + grp]) : off;
      const int code = static_cast<int>((word >> (4 * k)) & 0xFu) - zp;
      const float sc = __half2float(__ushort_as_half(scales16[r * ngroups + grp]));
      float what = static_cast<float>(code) * sc;
      if (s) what = __fdiv_rn(what, sv[k]);
      d32[k] = wv[k] - what;
    }
    if (dW32) {
      float4* dst = reinterpret_cast<float4*>(dW32 + r * in + wd * 8);
      dst[0] = make_float4(d32[0], d32[1], d32[2], d32[3]);
      dst[1] = make_float4(d32[4], d32[5], d32[6], d32[7]);
      continue;
    }
    uint4 o;
    o.x = floats_to_bf16x2_bits(d32[0], d32[1]);
    o.y = floats_to_bf16x2_bits(d32[2], d32[3]);
    o.z = floats_to_bf16x2_bits(d32[4], d32[5]);
    o.w = floats_to_bf16x2_bits(d32[6], d32[7]);
    *reinterpret_cast<uint4*>(dW + r * in + wd * 8) = o;
  }
}

unsigned grid_for(int64_t work, int threads) {
  DeviceInfo info;
  int sms = (device_info(&info) == PIQ_OK) ? info.sm_count : 148;
  const int64_t want = ceil_div(work, threads);
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(want, 16LL * sms)));
}

int last_error() { return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA; }

}  // namespace

// Row splits of the column-statistics pass: about 1024 CTAs in all, at least 64
// rows each.  Device-independent, so workspace queries can use it.
int colstats_splits(int64_t n, int64_t in) {
  const int64_t col_blocks = ceil_div(in, 256);
  int64_t splits = std::min<int64_t>(ceil_div(1024, col_blocks), ceil_div(n, 64));
  return static_cast<int>(std::max<int64_t>(1, splits));
}

int launch_colstats(const uint16_t* X, int64_t n, int64_t in, double* partials, int splits,
                    double* mean_abs, double* sumsq, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(ceil_div(in, 256)), static_cast<unsigned>(splits));
  const unsigned fgrid = static_cast<unsigned>(ceil_div(in, 256));
  if (mean_abs) {
    note_launch();
    colstats_kernel<0><<<grid, 256, 0, stream>>>(X, n, in, splits, partials);
    note_launch();
    colstats_finish_kernel<<<fgrid, 256, 0, stream>>>(partials, n, in, splits, 1, mean_abs);
  }
  if (sumsq) {
    note_launch();
    colstats_kernel<1><<<grid, 256, 0, stream>>>(X, n, in, splits, partials);
    note_launch();
    colstats_finish_kernel<<<fgrid, 256, 0, stream>>>(partials, n, in, splits, 0, sumsq);
  }
  return last_error();
}

int launch_gather_columns(const float* W, int64_t out, int64_t in, const int32_t* perm,
                          const float* cs, float* Wq, cudaStream_t stream) {
  if (in % 4 != 0 || (reinterpret_cast<uintptr_t>(W) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(Wq) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(perm) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(cs) & 15u) != 0)
    return PIQ_ERR_INVALID_ARG;
  note_launch();
  gather_columns_kernel<<<grid_for(out * in / 4, 256), 256, 0, stream>>>(W, out, in, perm, cs,
                                                                         Wq);
  return last_error();
}

int launch_scale_upper(float* H, int64_t in, const float* s, DeviceStatus* st,
                       cudaStream_t stream) {
  if (in % 4 != 0 || (reinterpret_cast<uintptr_t>(H) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(s) & 15u) != 0 || s == nullptr)
    return PIQ_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(in / 4, 256), 16)),
            static_cast<unsigned>(std::min<int64_t>(in, 65535)));
  note_launch();
  scale_upper_kernel<<<grid, 256, 0, stream>>>(H, in, s, st);
  return last_error();
}

int launch_scale_upper(double* H, int64_t in, const float* s, DeviceStatus* st,
                       cudaStream_t stream) {
  if (s == nullptr) return PIQ_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(in, 256), 16)),
            static_cast<unsigned>(std::min<int64_t>(in, 65535)));
  note_launch();
  scale_upper64_kernel<<<grid, 256, 0, stream>>>(H, in, s, st);
  return last_error();
}

int launch_scale_sumsq(double* sumsq, int64_t in, const float* s, cudaStream_t stream) {
  note_launch();
  scale_sumsq_kernel<<<static_cast<unsigned>(ceil_div(in, 256)), 256, 0, stream>>>(sumsq, in, s);
  return last_error();
}

int launch_pack(const int8_t* codes, const float* qscale, const uint8_t* qzero,
                const int32_t* invperm, int64_t out, int64_t in, int bits, int g,
                const float* W0, const float* cs, uint32_t* qweight, uint16_t* scales16,
                uint16_t* dW, float* dW32, int32_t* g_idx, cudaStream_t stream) {
  if ((dW != nullptr || dW32 != nullptr) && W0 == nullptr) return PIQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cs) & 15u) != 0) return PIQ_ERR_INVALID_ARG;
  note_launch();
  pack_kernel<<<grid_for(out * (in / 8), 256), 256, 0, stream>>>(
      codes, qscale, qzero, invperm, out, in, bits, g, W0, cs, qweight, scales16, dW, dW32,
      g_idx);
  return last_error();
}

int launch_awq_scale_table(const double* mean_abs, int64_t in, const float* alphas_dev,
                           int n_alpha, float* s_table, cudaStream_t stream) {
  note_launch();
  awq_scale_table_kernel<<<grid_for(n_alpha * in, 256), 256, 0, stream>>>(mean_abs, in,
                                                                          alphas_dev, n_alpha,
                                                                          s_table);
  return last_error();
}

int launch_awq_delta(const float* W, int64_t out, int64_t in, int bits, int g,
                     const float* s_table, int n_alpha, uint16_t* dW, cudaStream_t stream) {
  const int64_t warps = out * ceil_div(in, g);
  note_launch();
  const bool pow2 = g >= 8 && g <= 256 && (g & (g - 1)) == 0;
  if (pow2 && in % 8 == 0) {
    const int64_t rwarps = ceil_div(out, kRows) * ceil_div(in, 256);
    awq_delta_rows_kernel<<<grid_for(rwarps * 32, 256), 256, 0, stream>>>(W, out, in, bits, g,
                                                                          s_table, n_alpha, dW);
  } else if (g % 4 == 0 && g <= 128)
    awq_delta_vec_kernel<<<grid_for(warps * 32, 256), 256, 0, stream>>>(W, out, in, bits, g,
                                                                        s_table, n_alpha, dW);
  else
    awq_delta_kernel<<<grid_for(warps * 32, 256), 256, 0, stream>>>(W, out, in, bits, g, s_table,
                                                                     n_alpha, dW);
  return last_error();
}

int launch_group_quant(const float* W, int64_t out, int64_t in, int bits, int g,
                       const float* s_table, const int* sel, int8_t* codes, float* qscale,
                       float* s_out, cudaStream_t stream) {
  const int64_t warps = out * ceil_div(in, g);
  note_launch();
  group_quant_kernel<<<grid_for(warps * 32, 256), 256, 0, stream>>>(W, out, in, bits, g, s_table,
                                                                     sel, codes, qscale, s_out);
  return last_error();
}

int launch_argmin(const double* err, int n, const float* alphas_dev, int* best_idx,
                  float* best_alpha, cudaStream_t stream) {
  note_launch();
  argmin_kernel<<<1, 32, 0, stream>>>(err, n, alphas_dev, best_idx, best_alpha);
  return last_error();
}

int launch_dequant_delta(const float* W, int64_t out, int64_t in, const uint32_t* qweight,
                         const uint16_t* scales16, const uint8_t* zeros, const int32_t* g_idx,
                         const float* s, int bits, int g, uint16_t* dW, float* dW32,
                         DeviceStatus* st, cudaStream_t stream) {
  if ((dW == nullptr) == (dW32 == nullptr)) return PIQ_ERR_INVALID_ARG;
  note_launch();
  dequant_delta_kernel<<<grid_for(out * (in / 8), 256), 256, 0, stream>>>(
      W, out, in, qweight, scales16, zeros, g_idx, s, bits, g, dW, dW32, st);
  return last_error();
}

}  // namespace piq
