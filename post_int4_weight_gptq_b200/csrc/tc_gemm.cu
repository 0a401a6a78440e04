// Tensor-core GEMMs on sm_100a: tcgen05.mma (kind::f16, bf16 x bf16 -> fp32 in
// TMEM), operands staged in shared memory by TMA (128-byte swizzle), one
// persistent CTA per SM.
//
//   * syrk_xtx   H = X^T X, the proxy Hessian of "GPTQ versus AWQ objectives"
//                ("A strong answer", listing: H = X.T @ X).  X[n, in] is
//                row-major, so both operands are MN-major tiles (the sample
//                index n is the contraction).  Only tiles touching the upper
//                triangle are computed.  The sample range is cut into chunks of
//                KC samples: each chunk's fp32 tile leaves TMEM and is added into
//                H by a TMA reduce (the first chunk stores), one chunk after the
//                other by the CTA that owns the tile, so the sum is deterministic
//                and the tensor-core accumulation error grows with KC rather
//                than with n.
//   * err_sumsq  E_b = ||X D_b^T||_F^2 for stacked D_b (D = W - What), the
//                shared objective of both methods ("How to approach it").  Both
//                operands are K-major; the epilogue squares and sums the
//                accumulator straight out of TMEM, so the [n, out] product
//                never reaches memory.  One double per tile, reduced later in a
//                fixed order (deterministic).
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into a 4-stage
// ring; warp 1 lane 0 issues the MMAs and commits; warps 2..5 drain one of two
// 256-column accumulators while the MMA warp fills the other.  Every wait is
// bounded (common.cuh); no multicast loads are used.
#include <cuda.h>

#include <mutex>

#include "internal.h"

namespace piq {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;               // two fp32 accumulators
constexpr int GROUP_M = 16;                     // raster group (err_sumsq)
// Samples per TMEM accumulation before the tile is flushed into H.  The
// relative error of the tensor-core fp32 sum grows about linearly with the
// number of MMAs accumulated in place; 4096 samples (256 MMAs of k = 16) keep
// it near 2e-5 of sqrt(H_ii H_jj) whatever n is.
constexpr int KC = 4096;
constexpr int STG_BYTES = 4 * 2 * 32 * 32 * 4;  // H epilogue: two 32x32 fp32 slabs per warp

enum { EPI_STORE_UPPER = 0, EPI_SUMSQ = 1 };

template <int EPI>
constexpr int smem_bytes() {
  return STAGES * STAGE_BYTES + (EPI == EPI_STORE_UPPER ? STG_BYTES : 0) + 1024 /*align*/ +
         256 /*barriers*/;
}

struct Params {
  int M, N, K;
  int m_tiles, n_tiles, batch;
  int num_tiles;
  float* C;
  int64_t ldc;
  int accumulate;
  int kb_chunk;  // k blocks per accumulation chunk (>= number of k blocks: one chunk)
  double* partials;
  DeviceStatus* st;
};

// Tile t -> (m tile, n tile, batch entry).
template <int EPI>
__device__ __forceinline__ void decode_tile(const Params& p, int t, int& mt, int& nt, int& bz) {
  if (EPI == EPI_STORE_UPPER) {
    // n-panel b holds m tiles a with a*BM < (b+1)*BN (they touch j >= i).
    int acc = 0;
    bz = 0;
    for (int b = 0; b < p.n_tiles; ++b) {
      int cnt = min(p.m_tiles, (int)(((int64_t)(b + 1) * BN + BM - 1) / BM));
      if (t < acc + cnt) {
        nt = b;
        mt = t - acc;
        return;
      }
      acc += cnt;
    }
    mt = nt = 0;
  } else {
    const int per = p.m_tiles * p.n_tiles;
    bz = t / per;
    const int r = t - bz * per;
    const int grp = r / (GROUP_M * p.n_tiles);
    const int first_m = grp * GROUP_M;
    const int gm = min(GROUP_M, p.m_tiles - first_m);
    const int w = r - grp * GROUP_M * p.n_tiles;
    mt = first_m + w % gm;
    nt = w / gm;
  }
}

template <bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* stg_all = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);  // H epilogue only
  uint64_t* full = reinterpret_cast<uint64_t*>(
      smem + STAGES * STAGE_BYTES + (EPI == EPI_STORE_UPPER ? STG_BYTES : 0));
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // an earlier step already failed: do nothing (uniform over the CTA)
  if (status_bad(p.st)) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI == EPI_STORE_UPPER) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.K + BK - 1) / BK;
  const int n_chunks = num_kb <= p.kb_chunk ? 1 : 1 + (num_kb - 1) / p.kb_chunk;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mt, nt, bz;
        decode_tile<EPI>(p, t, mt, nt, bz);
        const int m0 = mt * BM, n0 = nt * BN;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, p.st, 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
          const int k0 = kb * BK;
          if (A_MN) {
            tma_load_2d(sa, &tmA, &full[s], m0, k0);
            tma_load_2d(sa + 8192, &tmA, &full[s], m0 + 64, k0);
          } else {
            tma_load_2d(sa, &tmA, &full[s], k0, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_2d(sb + c * 8192, &tmB, &full[s], n0 + 64 * c, k0);
          } else {
            tma_load_3d(sb, &tmB, &full[s], k0, n0, bz);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        for (int ch = 0; ch < n_chunks && ok; ++ch, ++lt) {
          const int buf = lt & 1;
          const uint32_t use = static_cast<uint32_t>(lt >> 1);
          if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, p.st, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
          const int kb0 = ch * p.kb_chunk;
          const int kb1 = num_kb - kb0 <= p.kb_chunk ? num_kb : kb0 + p.kb_chunk;
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph, p.st, 3)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = A_MN ? smem_desc(a_addr + kk * 2048, 8192, 1024, kLayoutSw128)
                                       : smem_desc(a_addr + kk * 32, 16, 1024, kLayoutSw128);
              const uint64_t bd = B_MN ? smem_desc(b_addr + kk * 2048, 8192, 1024, kLayoutSw128)
                                       : smem_desc(b_addr + kk * 32, 16, 1024, kLayoutSw128);
              umma_bf16(d_tmem, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
            }
            umma_commit(&empty[s]);  // frees the stage once these MMAs finish
          }
          if (ok) umma_commit(&acc_full[buf]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int lt = 0;
    if (EPI == EPI_SUMSQ) {
      for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++lt) {
        const int buf = lt & 1;
        const uint32_t use = static_cast<uint32_t>(lt >> 1);
        if (!mbar_wait(&acc_full[buf], use & 1u, p.st, 4)) break;
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * BN);
        double acc = 0.0;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          float s = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) s = fmaf(v[i], v[i], s);
          acc += static_cast<double>(s);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        // one partial per (tile, lane quarter): no cross-warp synchronisation
        acc = warp_sum_d(acc);
        if (lane == 0) p.partials[static_cast<int64_t>(t) * 4 + q] = acc;
      }
    } else {
      // Each warp owns 32 rows of the tile and moves them out in 32x32 slabs
      // through a double-buffered staging tile in the TMA 128-byte swizzle
      // (16-byte chunk k of row r sits at chunk k ^ (r % 8)).  A chunk's slabs
      // are stored (first chunk, accumulate == 0) or reduce-added into H; the
      // next chunk of the same tile waits until they have all landed, so the
      // additions into H happen in chunk order.
      float* stg = stg_all + q * 2 * 1024;
      uint32_t nst = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mt, nt, bz;
        decode_tile<EPI>(p, t, mt, nt, bz);
        const int row0 = mt * BM + q * 32;
        for (int ch = 0; ch < n_chunks; ++ch, ++lt) {
          const int buf = lt & 1;
          const uint32_t use = static_cast<uint32_t>(lt >> 1);
          if (!mbar_wait(&acc_full[buf], use & 1u, p.st, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0 && ch > 0) bulk_wait_all();  // previous chunk's additions landed
          __syncwarp();
          const bool store = ch == 0 && p.accumulate == 0;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(buf * BN);
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            const int col0 = nt * BN + c * 32;
            // slabs wholly below the diagonal, or outside H, are not needed
            if (row0 >= p.M || col0 >= p.N || col0 + 32 <= row0) continue;
            float v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);  // lane = row, v[i] = column i
            float* sb = stg + (nst & 1) * 1024;
            if (lane == 0) bulk_wait_read<1>();  // this buffer's previous copy has read it
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<float4*>(sb + lane * 32 + ((k ^ (lane & 7)) << 2)) =
                  make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (store)
                tma_store_3d(&tmC, sb, col0, row0, 0);
              else
                tma_reduce_add_3d(&tmC, sb, col0, row0, 0);
              bulk_commit();
            }
            ++nst;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
      }
      if (lane == 0) bulk_wait_all();  // every copy of this warp has landed
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// -------------------------------------------------------------- host helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map (bf16 operands or the fp32 H), innermost dimension first, 128-byte swizzle.
int make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
             const uint64_t* strides_bytes, const uint32_t* box,
             CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return PIQ_ERR_CUDA;
  cuuint64_t d[3], s[2];
  cuuint32_t b[3], e[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUresult r = fn(map, type, rank, const_cast<void*>(base), d, s, b, e,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PIQ_OK : PIQ_ERR_INVALID_ARG;
}

template <bool A_MN, bool B_MN, int EPI>
int launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, const Params& p,
           cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  auto kern = tc_gemm_kernel<A_MN, B_MN, EPI>;
  constexpr int smem = smem_bytes<EPI>();
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  DeviceInfo info;
  int rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  const int grid = std::max(1, std::min(p.num_tiles, info.sm_count));
  note_launch();
  kern<<<grid, THREADS, smem, stream>>>(a, b, c, p);
  return cudaGetLastError() == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace

int launch_syrk_xtx(const uint16_t* X, int64_t n, int64_t in, float* H, int accumulate,
                    DeviceStatus* st, cudaStream_t stream) {
  if (n < 1 || in < 8 || in % 8 != 0 || n > INT32_MAX || in > INT32_MAX / 2)
    return PIQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) & 15u) != 0 || (reinterpret_cast<uintptr_t>(H) & 15u) != 0)
    return PIQ_ERR_INVALID_ARG;
  CUtensorMap map, mc;
  const uint64_t dims[2] = {static_cast<uint64_t>(in), static_cast<uint64_t>(n)};
  const uint64_t strides[1] = {static_cast<uint64_t>(in) * 2};
  const uint32_t box[2] = {64, 64};
  int rc = make_map(&map, X, 2, dims, strides, box);
  if (rc != PIQ_OK) return rc;
  {
    const uint64_t cd[3] = {static_cast<uint64_t>(in), static_cast<uint64_t>(in), 1};
    const uint64_t cs[2] = {static_cast<uint64_t>(in) * 4,
                            static_cast<uint64_t>(in) * static_cast<uint64_t>(in) * 4};
    const uint32_t cb[3] = {32, 32, 1};
    rc = make_map(&mc, H, 3, cd, cs, cb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
    if (rc != PIQ_OK) return rc;
  }
  Params p{};
  p.M = p.N = static_cast<int>(in);
  p.K = static_cast<int>(n);
  p.m_tiles = static_cast<int>(ceil_div(in, BM));
  p.n_tiles = static_cast<int>(ceil_div(in, BN));
  p.batch = 1;
  int total = 0;
  for (int b = 0; b < p.n_tiles; ++b)
    total += std::min(p.m_tiles, static_cast<int>(((int64_t)(b + 1) * BN + BM - 1) / BM));
  p.num_tiles = total;
  p.C = H;
  p.ldc = in;
  p.accumulate = accumulate;
  p.kb_chunk = KC / BK;
  p.st = st;
  return launch<true, true, EPI_STORE_UPPER>(map, map, mc, p, stream);
}

int64_t sumsq_partials_count(int64_t n, int64_t rows, int batch) {
  return ceil_div(n, BM) * ceil_div(rows, BN) * batch * 4;
}

int launch_err_sumsq(const uint16_t* X, int64_t n, int64_t in, const uint16_t* D, int64_t rows,
                     int batch, double* partials, DeviceStatus* st, cudaStream_t stream) {
  if (n < 1 || in < 8 || in % 8 != 0 || rows < 1 || batch < 1 || n > INT32_MAX ||
      rows > INT32_MAX)
    return PIQ_ERR_INVALID_ARG;
  CUtensorMap ma, mb;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(in), static_cast<uint64_t>(n)};
    const uint64_t strides[1] = {static_cast<uint64_t>(in) * 2};
    const uint32_t box[2] = {64, BM};
    int rc = make_map(&ma, X, 2, dims, strides, box);
    if (rc != PIQ_OK) return rc;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(in), static_cast<uint64_t>(rows),
                              static_cast<uint64_t>(batch)};
    const uint64_t strides[2] = {static_cast<uint64_t>(in) * 2,
                                 static_cast<uint64_t>(in) * static_cast<uint64_t>(rows) * 2};
    const uint32_t box[3] = {64, BN, 1};
    int rc = make_map(&mb, D, 3, dims, strides, box);
    if (rc != PIQ_OK) return rc;
  }
  Params p{};
  p.M = static_cast<int>(n);
  p.N = static_cast<int>(rows);
  p.K = static_cast<int>(in);
  p.m_tiles = static_cast<int>(ceil_div(n, BM));
  p.n_tiles = static_cast<int>(ceil_div(rows, BN));
  p.batch = batch;
  const int64_t total = static_cast<int64_t>(p.m_tiles) * p.n_tiles * batch;
  if (total > INT32_MAX) return PIQ_ERR_INVALID_ARG;
  p.num_tiles = static_cast<int>(total);
  p.partials = partials;
  p.kb_chunk = INT32_MAX;  // one accumulation per tile
  p.st = st;
  return launch<false, false, EPI_SUMSQ>(ma, mb, ma, p, stream);
}

// ------------------------------------------------ fixed-order partial reduction
namespace {
constexpr int RP_THREADS = 512;
// One block per batch entry.  Thread t sums the elements t, t + 512, ... in four
// interleaved accumulators (so four loads are in flight), then the block folds
// the per-thread sums in a fixed tree: the order never depends on timing.
__global__ void __launch_bounds__(RP_THREADS)
    reduce_partials_kernel(const double* partials, int64_t per, double* out) {
  __shared__ double sh[RP_THREADS];
  const double* src = partials + static_cast<int64_t>(blockIdx.x) * per;
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  int64_t i = threadIdx.x;
  for (; i + 3 * RP_THREADS < per; i += 4 * RP_THREADS) {
    a0 += src[i];
    a1 += src[i + RP_THREADS];
    a2 += src[i + 2 * RP_THREADS];
    a3 += src[i + 3 * RP_THREADS];
  }
  for (; i < per; i += RP_THREADS) a0 += src[i];
  sh[threadIdx.x] = (a0 + a1) + (a2 + a3);
  __syncthreads();
  for (int s = RP_THREADS / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[blockIdx.x] = sh[0];
}
}  // namespace

int launch_reduce_partials(const double* partials, int64_t n, int64_t rows, int batch,
                           double* out, cudaStream_t stream) {
  const int64_t per = ceil_div(n, BM) * ceil_div(rows, BN) * 4;
  note_launch();
  reduce_partials_kernel<<<batch, RP_THREADS, 0, stream>>>(partials, per, out);
  return cudaGetLastError() == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace piq
