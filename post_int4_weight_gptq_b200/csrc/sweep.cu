// GPTQ column sweep, block by block.
//
// "GPTQ versus AWQ objectives", section "A strong answer", listing loop body:
// at each group start (j % g == 0) a per-row scale max|W[:, j:j+g]| / qmax from
// the current, already updated W; Q[:, j] = clip(round(W[:, j] / scale),
// -qmax-1, qmax) * scale; err = (W[:, j] - Q[:, j]) / U[j, j]; every later column
// gets W[:, k] -= err * U[j, k].  The remark after the listing batches the
// updates over column blocks: inside a block the updates are applied at once
// (here, in registers), and the block's errors update all later columns with
// one GEMM, W[:, e:] -= Err[:, b:e] U[b:e, e:] (simt_gemm.cu).
//
// Blocks are at most 128 wide and are cut so that every group start is either
// a block start or has its whole group inside its block; a group scale then
// only reads columns whose updates are all applied (g | 128, 128 | g, or any
// other g), so the arithmetic is the listing's.
//
// Kernel layout: one warp per ROWS rows; lane l holds columns l, l+32, l+64,
// l+96 of its rows in registers; U[b:e, b:e] sits in shared memory.  Column j
// is broadcast from its owner lane with a shuffle; the division W/scale is IEEE
// round-to-nearest and rintf rounds half to even (the listing's np.round).
#include <algorithm>
#include <vector>

#include "internal.h"

namespace piq {

namespace {

constexpr int B = kSweepB;    // 128
constexpr int ROWS = 2;       // rows per warp
constexpr int WARPS = 8;
constexpr int LDU = B + 1;

__global__ void __launch_bounds__(WARPS * 32)
    sweep_block_kernel(float* __restrict__ W, int64_t out, int64_t in, const float* __restrict__ U,
                       int64_t b, int kb, int bits, int g, int8_t* __restrict__ codes,
                       float* __restrict__ qscale, float* __restrict__ Err, DeviceStatus* st) {
  extern __shared__ float Us[];  // [kb][LDU]
  if (status_bad(st)) return;
  for (int idx = threadIdx.x; idx < kb * kb; idx += blockDim.x) {
    const int r = idx / kb, c = idx % kb;
    Us[r * LDU + c] = (c >= r) ? U[(b + r) * in + b + c] : 0.f;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * WARPS + warp) * ROWS;
  if (row0 >= out) return;
  const int qmax = (1 << (bits - 1)) - 1;
  const float fqmax = static_cast<float>(qmax);
  const float cmin = static_cast<float>(-qmax - 1), cmax = static_cast<float>(qmax);
  const int64_t ngroups = (in + g - 1) / g;

  float w[ROWS][4], e[ROWS][4], sc[ROWS];
  int cq[ROWS][4];
  bool valid[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    valid[r] = row0 + r < out;
    sc[r] = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = 32 * t + lane;
      w[r][t] = (valid[r] && c < kb) ? W[(row0 + r) * in + b + c] : 0.f;
      e[r][t] = 0.f;
      cq[r][t] = 0;
    }
  }
  // scale of a group that started before this block (b not a group start)
  if (b % g != 0) {
    const int64_t grp = b / g;
#pragma unroll
    for (int r = 0; r < ROWS; ++r) sc[r] = valid[r] ? qscale[(row0 + r) * ngroups + grp] : 0.f;
  }

#pragma unroll
  for (int s = 0; s < 4; ++s) {
#pragma unroll 4
    for (int o = 0; o < 32; ++o) {
      const int j = 32 * s + o;
      if (j >= kb) break;
      const int64_t p = b + j;
      if (p % g == 0) {  // group start: scale from the current weights
        const int64_t gend = std::min<int64_t>(p + g, in);
        const int jend = static_cast<int>(std::min<int64_t>(gend - b, kb));
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
          float m = 0.f;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int c = 32 * t + lane;
            if (c >= j && c < jend) m = fmaxf(m, fabsf(w[r][t]));
          }
          if (gend > b + kb && valid[r]) {  // group runs past the block: current W in memory
            const float* src = W + (row0 + r) * in;
            for (int64_t c = b + kb + lane; c < gend; c += 32) m = fmaxf(m, fabsf(src[c]));
          }
          m = warp_max(m);
          sc[r] = __fdiv_rn(m, fqmax);
          if (lane == 0 && valid[r]) qscale[(row0 + r) * ngroups + p / g] = sc[r];
        }
      }
      const float ujj = Us[j * LDU + j];
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const float wj = __shfl_sync(0xffffffffu, w[r][s], o);
        float q = 0.f;
        if (sc[r] > 0.f) q = fminf(fmaxf(rintf(__fdiv_rn(wj, sc[r])), cmin), cmax);
        const float err = __fdiv_rn(wj - q * sc[r], ujj);
        if (lane == o) {
          cq[r][s] = static_cast<int>(q);
          e[r][s] = err;
        }
#pragma unroll
        for (int t = s; t < 4; ++t) {
          const int c = 32 * t + lane;
          if (c > j) w[r][t] = fmaf(-err, Us[j * LDU + c], w[r][t]);
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    if (!valid[r]) continue;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int c = 32 * t + lane;
      if (c < kb) {
        codes[(row0 + r) * in + b + c] = static_cast<int8_t>(cq[r][t]);
        Err[(row0 + r) * B + c] = e[r][t];
      }
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
                   int8_t* codes, float* qscale, float* Err, DeviceStatus* st,
                   cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  const int smem = B * LDU * static_cast<int>(sizeof(float));
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(sweep_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  std::vector<std::pair<int64_t, int64_t>> blocks;
  block_partition(in, g, &blocks);
  const int64_t rows_per_cta = WARPS * ROWS;
  const unsigned grid = static_cast<unsigned>(ceil_div(out, rows_per_cta));
  for (const auto& be : blocks) {
    const int64_t b = be.first, e = be.second;
    const int kb = static_cast<int>(e - b);
    note_launch();
    sweep_block_kernel<<<grid, WARPS * 32, smem, stream>>>(Wq, out, in, U, b, kb, bits, g, codes,
                                                           qscale, Err, st);
    if (cudaGetLastError() != cudaSuccess) return PIQ_ERR_CUDA;
    if (e < in) {
      // W[:, e:] -= Err[:, :kb] U[b:e, e:]
      int rc = launch_simt_gemm(static_cast<int>(out), static_cast<int>(in - e), kb, -1.f, Err, B,
                                U + b * in + e, in, false, 1.f, Wq + e, in, 0, st, stream);
      if (rc != PIQ_OK) return rc;
    }
  }
  return PIQ_OK;
}

}  // namespace piq
