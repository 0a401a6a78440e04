// H = X^T X with FP64 sums, on the tcgen05 tensor cores (kind::f16, bf16 x bf16).
//
// "GPTQ versus AWQ objectives", section "A strong answer" (listing:
// H = X.T @ X, the proxy Hessian).  Every bf16 x bf16 product is exact in FP32;
// what rounds is the accumulation.  The tensor core adds the products of each
// MMA (16 samples) to its FP32 TMEM accumulator with one rounding toward zero,
// so a long TMEM accumulation drifts (at 32768 samples, 1024-sample TMEM
// chunks bias diag(H) by -1.9e-6 relative), and an FP32 running sum of chunks
// adds a random walk on top.  At a 28672-column layer either flips enough GPTQ
// rounding decisions to break the code parity with an FP64 evaluation of the
// loop.  Here each 128-sample chunk (8 MMAs) is accumulated in TMEM; two
// consecutive chunks are added in FP32 (round to nearest) and that sum goes
// into FP64 sums held in the epilogue threads' registers, in chunk order.  The
// FP32 roundings left are those inside a chunk and one per chunk pair; the
// pairing halves the fp32 -> fp64 conversions, which run at a quarter of the
// FP32 rate and would otherwise set the pace.  Four 128-column TMEM
// accumulators: the MMA warp fills one pair while the epilogue drains the
// other.
//
// Tiles of 128 x 128 on or above the diagonal (the fp64 sums of a 128 x 256
// tile would not fit in registers), round-robin over one persistent CTA per
// SM, so all CTAs sweep the same sample range together and X streams through
// L2 once per wave.  X[n, in] is row-major, so both operands are MN-major
// tiles (two 64-column TMA boxes each, 128-byte swizzle).  Output: the upper
// triangle of H as fp64 (entries below the diagonal inside diagonal tiles are
// written too; nothing reads them).
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads into a 7-stage ring;
// warp 1 lane 0 issues the MMAs; warps 2..9 drain one of two 128-column TMEM
// accumulators (warp w reads lanes 32 (w % 4) .. and columns 64 ((w - 2) / 4) ..)
// while the MMA warp fills the other.  Every wait is bounded; no multicast loads.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "internal.h"

namespace piq {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 64;
constexpr int STAGES = 7;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int NBUF = 4;  // TMEM accumulators (two chunk pairs)
constexpr int TMEM_COLS = NBUF * BN;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
static_assert(SMEM_BYTES <= 227 * 1024, "pipeline exceeds shared memory");
constexpr int KC = 128;  // samples per TMEM accumulation
constexpr int KB_CHUNK = KC / BK;

struct S64Params {
  int in, n;
  int tiles_1d, num_tiles;
  double* H;
  DeviceStatus* st;
};

// Tile t -> (mt, nt) with mt <= nt.  The upper triangle of tiles is walked in
// super-blocks of G x G tiles (super-column by super-column; inside a
// super-column the blocks above the diagonal, then the diagonal one), row by
// row inside a block.  One wave of persistent CTAs (148 tiles) then covers
// about one super-block, i.e. 2 G column blocks of X, each read from HBM once
// and shared by G tiles through L2; column panel by column panel a wave would
// touch ~150 column blocks and use each once.
constexpr int kSuperTile = 12;

__device__ __forceinline__ void tile_of(int t, int T, int& mt, int& nt) {
  constexpr int G = kSuperTile;
  int acc = 0;
  for (int J = 0; J * G < T; ++J) {
    const int c = min(G, T - J * G);  // tile columns of super-column J
    const int above = c * G * J;      // tiles of its blocks above the diagonal
    const int cnt = above + c * (c + 1) / 2;
    if (t < acc + cnt) {
      int li = t - acc;
      if (li < above) {
        const int I = li / (G * c);
        const int r = li - I * G * c;
        mt = I * G + r / c;
        nt = J * G + r % c;
      } else {
        li -= above;
        int b = static_cast<int>((sqrtf(8.f * static_cast<float>(li) + 1.f) - 1.f) * 0.5f);
        while ((b + 1) * (b + 2) / 2 <= li) ++b;
        while (b * (b + 1) / 2 > li) --b;
        mt = J * G + (li - b * (b + 1) / 2);
        nt = J * G + b;
      }
      return;
    }
    acc += cnt;
  }
  mt = nt = 0;
}

__global__ void __launch_bounds__(THREADS, 1)
    syrk64_kernel(const __grid_constant__ CUtensorMap tmX, S64Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [NBUF]
  uint64_t* acc_empty = acc_full + NBUF;  // [NBUF]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + NBUF);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.n + BK - 1) / BK;
  const int n_chunks = (num_kb + KB_CHUNK - 1) / KB_CHUNK;
  pdl_wait();
  const bool skip = status_bad(p.st);

  if (skip) {
  } else if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_of(t, p.tiles_1d, mt, nt);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, p.st, 51)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          const int k0 = kb * BK;
          tma_load_2d(sa, &tmX, &full[s], mt * BM, k0);
          tma_load_2d(sa + 8192, &tmX, &full[s], mt * BM + 64, k0);
          tma_load_2d(sb, &tmX, &full[s], nt * BN, k0);
          tma_load_2d(sb + 8192, &tmX, &full[s], nt * BN + 64, k0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, true, true);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        for (int ch = 0; ch < n_chunks && ok; ++ch, ++lt) {
          const int buf = lt % NBUF;
          const uint32_t use = static_cast<uint32_t>(lt / NBUF);
          if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, p.st, 52)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
          const int kb0 = ch * KB_CHUNK;
          const int kb1 = std::min(num_kb, kb0 + KB_CHUNK);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph, p.st, 53)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = smem_desc(a_addr + kk * 2048, 8192, 1024, kLayoutSw128);
              const uint64_t bd = smem_desc(b_addr + kk * 2048, 8192, 1024, kLayoutSw128);
              umma_bf16(d_tmem, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
            }
            umma_commit(&empty[s]);
          }
          if (ok) umma_commit(&acc_full[buf]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;  // column half: 64 columns
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      int mt, nt;
      tile_of(t, p.tiles_1d, mt, nt);
      const int row0 = mt * BM + q * 32;
      const int colh = nt * BN + h * 64;
      // a 32-column slab wholly below the diagonal is never stored
      const bool live0 = colh + 32 > row0 && colh < p.in && row0 < p.in;
      const bool live1 = colh + 64 > row0 && colh + 32 < p.in && row0 < p.in;
      double sum[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) sum[i] = 0.0;
      // chunks in pairs (a tile with an odd count ends with a single one);
      // chunk ch sits in buffer (tile's first chunk index + ch) % NBUF
      for (int ch = 0; ch < n_chunks; ch += 2) {
        const int two = (ch + 1 < n_chunks) ? 2 : 1;
        uint32_t taddr[2];
        for (int u = 0; u < two; ++u) {
          const int l = lt + ch + u;
          const int buf = l % NBUF;
          const uint32_t use = static_cast<uint32_t>(l / NBUF);
          if (!mbar_wait(&acc_full[buf], use & 1u, p.st, 54)) {
            ok = false;
            break;
          }
          taddr[u] = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                     static_cast<uint32_t>(buf * BN + h * 64);
        }
        if (!ok) break;
        tc_fence_after();
        // 16 columns per TMEM load keep the fp64 sums and the loaded values
        // within the register budget of ten warps per SM
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          if (qq < 2 ? live0 : live1) {
            float v[16];
            tmem_ld_32x32b_x16(taddr[0] + 16 * qq, v);
            if (two == 2) {
              float w[16];
              tmem_ld_32x32b_x16(taddr[1] + 16 * qq, w);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(v[i], w[i]);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) sum[16 * qq + i] += static_cast<double>(v[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int u = 0; u < two; ++u) mbar_arrive(&acc_empty[(lt + ch + u) % NBUF]);
      }
      lt += n_chunks;
      if (!ok) break;
      const int row = row0 + lane;
      if (row < p.in) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col0 = colh + 32 * c;
          if ((c == 0 ? !live0 : !live1) || col0 >= p.in) continue;
          double* dst = p.H + static_cast<int64_t>(row) * p.in + col0;
          if (col0 + 32 <= p.in) {
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              *reinterpret_cast<double2*>(dst + i) = make_double2(sum[32 * c + i], sum[32 * c + i + 1]);
          } else {
            const int lim = p.in - col0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < lim) dst[i] = sum[32 * c + i];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_s64() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

}  // namespace

int launch_syrk64(const uint16_t* X, int64_t n, int64_t in, double* H, DeviceStatus* st,
                  cudaStream_t stream) {
  if (n < 1 || in < 8 || in % 8 != 0 || n > INT32_MAX || in > (1 << 20)) return PIQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) & 15u) || (reinterpret_cast<uintptr_t>(H) & 15u))
    return PIQ_ERR_INVALID_ARG;
  EncodeTiledFn fn = encode_fn_s64();
  if (fn == nullptr) return PIQ_ERR_CUDA;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(in), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(in) * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return PIQ_ERR_INVALID_ARG;
  S64Params p{};
  p.in = static_cast<int>(in);
  p.n = static_cast<int>(n);
  p.tiles_1d = static_cast<int>(ceil_div(in, BM));
  const int64_t tot = static_cast<int64_t>(p.tiles_1d) * (p.tiles_1d + 1) / 2;
  if (tot > INT32_MAX) return PIQ_ERR_INVALID_ARG;
  p.num_tiles = static_cast<int>(tot);
  p.H = H;
  p.st = st;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(syrk64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  DeviceInfo info;
  int rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  const int grid = std::max(1, std::min(p.num_tiles, info.sm_count));
  note_launch();
  if (launch_pdl(syrk64_kernel, dim3(grid), dim3(THREADS), SMEM_BYTES, stream, map, p) !=
      cudaSuccess)
    return PIQ_ERR_CUDA;
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace piq
