// FP32-accurate GEMM on the tcgen05 tensor cores (kind::tf32, three passes).
//
// The FP32 products of the path (the GPTQ trailing update W[:, e:] -= Err U and
// the panel updates of the Cholesky and the triangular inverse that produce U)
// need about FP32 accuracy; a single TF32 pass (10-bit mantissa) is too coarse.
// Each operand is split into x = hi + lo with hi = x with its 13 low mantissa
// bits cleared and lo = x - hi (exact in fp32).  The tensor core reads only the
// top 19 bits of a 32-bit operand, so the TMA-landed tile itself serves as hi
// and only lo is written; the tile is accumulated in TMEM as
// A_hi B_hi + A_hi B_lo + A_lo B_hi  (lo is itself cut to 19 bits by the
// tensor core, and the dropped A_lo B_lo is ~2^-20 of the product).  A_hi B_hi
// and the two cross terms go to separate accumulators, added in the epilogue:
// the fp32 TMEM sum truncates relative to its own magnitude, so the small
// terms would otherwise lose their precision against the large one (this
// matters over the hundreds of panel updates of a 28672-wide factor).
//
// C = alpha A op(B) + beta C, all fp32 row-major: A [M][K] (K-major tiles), B
// [K][N] (MN-major tiles) or, with trans_b, [N][K] (K-major).  Modes: 0 plain;
// 1 only tiles touching the lower triangle of C; 2 A lower triangular; 3 B lower
// used transposed; 4 B lower used as is (zero K ranges are skipped per tile).
// Batched over entries with element strides; entry z may have fewer rows.
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads of fp32 tiles into a
// 3-stage ring; warps 6..9 write the lo part of each landed tile; warp 1 lane 0
// issues the MMAs; warps 2..5 drain one of two accumulator pairs.  Every
// wait is bounded; no multicast loads.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "internal.h"

namespace piq {

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 32;                       // fp32 elements = one 128-byte row
constexpr int STAGES = 3;
constexpr int TILE_BYTES = BM * BK * 4;      // 16 KB (A and B tiles are the same size)
constexpr int STAGE_BYTES = 4 * TILE_BYTES;  // A_hi, B_hi, A_lo, B_lo
constexpr int THREADS = 320;
// two buffers x (hi.hi accumulator, cross-term accumulator) of BN columns
constexpr int TMEM_COLS = 4 * BN;
constexpr int TR_BYTES = 4 * 2 * 32 * 32 * 4;  // epilogue staging: 2 per epilogue warp
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + TR_BYTES + 1024 + 256;

struct SgParams {
  int M, N, K;
  float alpha, beta;
  float* C;
  int64_t ldc;
  int mode;
  bool trans_b;
  int m_tiles, n_tiles, tiles_per_z, num_tiles;
  int batch;
  int64_t stride_c;
  int64_t m_total, m_step;
  bool k_follows_m;
  bool reduce_add;  // beta == 1: C += alpha A op(B) by TMA reduce-add; else C = alpha A op(B)
  DeviceStatus* st;
};

struct TileInfo {
  int z, mt, nt;
  int M, K;      // this batch entry's rows and contraction length
  int kb0, kb1;  // k-block range [kb0, kb1) that can be nonzero
};

// Tile t -> entry, position and K range (identical in every warp role).
__device__ __forceinline__ TileInfo tile_info(const SgParams& p, int t) {
  TileInfo ti;
  ti.z = t / p.tiles_per_z;
  const int r = t - ti.z * p.tiles_per_z;
  if (p.mode == 1) {  // lower-triangular tile numbering: row mt has tiles 0..mt
    int mt = static_cast<int>((sqrtf(8.f * r + 1.f) - 1.f) * 0.5f);
    while ((mt + 1) * (mt + 2) / 2 <= r) ++mt;
    while (mt * (mt + 1) / 2 > r) --mt;
    ti.mt = mt;
    ti.nt = r - mt * (mt + 1) / 2;
  } else {
    ti.mt = r / p.n_tiles;
    ti.nt = r - ti.mt * p.n_tiles;
  }
  ti.M = p.M;
  ti.K = p.K;
  if (p.m_total > 0) {
    const int64_t mz = p.m_total - static_cast<int64_t>(ti.z) * p.m_step;
    if (mz < ti.M) ti.M = static_cast<int>(mz < 0 ? 0 : mz);
    if (p.k_follows_m) ti.K = ti.M;
  }
  const int m0 = ti.mt * BM, n0 = ti.nt * BN;
  int kend = ti.K, kbeg = 0;
  if (p.mode == 2) kend = min(kend, m0 + BM);
  if (p.mode == 3) kend = min(kend, n0 + BN);
  if (p.mode == 4) kbeg = min(kend, n0);
  if (m0 >= ti.M) kend = kbeg;  // empty tile of a short entry
  ti.kb0 = kbeg / BK;
  ti.kb1 = (kend + BK - 1) / BK;
  if (ti.kb1 < ti.kb0) ti.kb1 = ti.kb0;
  return ti;
}

// Instruction descriptor: kind::tf32, fp32 accumulate, M = 128, N = 128.
__host__ __device__ constexpr uint32_t idesc_tf32(bool b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}

__global__ void __launch_bounds__(THREADS, 1)
    tf32x3_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC, SgParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* tr = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);  // epilogue staging
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + TR_BYTES);
  uint64_t* split = full + STAGES;     // converters done with the stage
  uint64_t* empty = split + STAGES;    // MMAs done with the stage
  uint64_t* acc_full = empty + STAGES; // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&split[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // inputs come from the previous kernel; an earlier failure skips the work
  // (uniform over the CTA, which still frees its TMEM below)
  pdl_wait();
  const bool skip = status_bad(p.st);

  if (skip) {
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(p, t);
        const int m0 = ti.mt * BM, n0 = ti.nt * BN;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, p.st, 11)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + TILE_BYTES;
          mbar_arrive_expect_tx(&full[s], 2 * TILE_BYTES);
          const int k0 = kb * BK;
          tma_load_3d(sa, &tmA, &full[s], k0, m0, ti.z);
          if (p.trans_b) {
            tma_load_3d(sb, &tmB, &full[s], k0, n0, ti.z);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
              tma_load_3d(sb + c * (BK * 128), &tmB, &full[s], n0 + 32 * c, k0, ti.z);
          }
        }
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------- hi/lo split
    const int ct = threadIdx.x - 6 * 32;  // 0..127
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      const TileInfo ti = tile_info(p, t);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph, p.st, 12)) {
          ok = false;
          break;
        }
        uint4* hi = reinterpret_cast<uint4*>(smem + s * STAGE_BYTES);
        uint4* lo = reinterpret_cast<uint4*>(smem + s * STAGE_BYTES + 2 * TILE_BYTES);
        // a short last k-block of a batch entry: the map's K extent is the largest
        // entry's, so columns past this entry's K must be zeroed here
        const int klim = ti.K - kb * BK;
#pragma unroll 4
        for (int i = ct; i < 2 * TILE_BYTES / 16; i += 128) {
          uint4 v = hi[i];
          if (klim < BK) {
            const bool in_b = i >= TILE_BYTES / 16;
            const int j = in_b ? i - TILE_BYTES / 16 : i;
            if (!in_b || p.trans_b) {  // K-major tile: row of 32 k, chunks swizzled by row
              const int row = j >> 3;
              const int kc = ((j & 7) ^ (row & 7)) * 4;
              if (kc + 0 >= klim) v.x = 0u;
              if (kc + 1 >= klim) v.y = 0u;
              if (kc + 2 >= klim) v.z = 0u;
              if (kc + 3 >= klim) v.w = 0u;
            } else {  // MN-major tile: 4 boxes of 32 k-rows x 32 n
              const int krow = (j & 255) >> 3;
              if (krow >= klim) v = make_uint4(0u, 0u, 0u, 0u);
            }
          }
          uint4 h, l;
          h.x = v.x & 0xFFFFE000u;
          h.y = v.y & 0xFFFFE000u;
          h.z = v.z & 0xFFFFE000u;
          h.w = v.w & 0xFFFFE000u;
          l.x = __float_as_uint(__uint_as_float(v.x) - __uint_as_float(h.x));
          l.y = __float_as_uint(__uint_as_float(v.y) - __uint_as_float(h.y));
          l.z = __float_as_uint(__uint_as_float(v.z) - __uint_as_float(h.z));
          l.w = __float_as_uint(__uint_as_float(v.w) - __uint_as_float(h.w));
          if (klim < BK) hi[i] = v;  // a short k block: the zeroed columns
          lo[i] = l;
        }
        fence_proxy_async_smem();  // generic writes -> visible to the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive(&split[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_tf32(!p.trans_b);
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++lt) {
        const TileInfo ti = tile_info(p, t);
        const int buf = lt & 1;
        const uint32_t use = static_cast<uint32_t>(lt >> 1);
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, p.st, 13)) break;
        tc_fence_after();
        // hi.hi and the cross terms accumulate apart: the small terms then keep
        // their precision (the fp32 TMEM sum truncates relative to its own size)
        const uint32_t d_big = tmem_base + static_cast<uint32_t>(buf * 2 * BN);
        const uint32_t d_small = d_big + BN;
        bool first = true;
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&split[s], ph, p.st, 14)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_hi = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_hi = a_hi + TILE_BYTES;
          const uint32_t a_lo = a_hi + 2 * TILE_BYTES;
          const uint32_t b_lo = a_hi + 3 * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            const uint64_t ah = smem_desc(a_hi + kk * 32, 16, 1024, kLayoutSw128);
            const uint64_t al = smem_desc(a_lo + kk * 32, 16, 1024, kLayoutSw128);
            uint64_t bh, bl;
            if (p.trans_b) {
              bh = smem_desc(b_hi + kk * 32, 16, 1024, kLayoutSw128);
              bl = smem_desc(b_lo + kk * 32, 16, 1024, kLayoutSw128);
            } else {
              // MN-major 32-bit operands use the 128-byte swizzle with 32-byte atoms:
              // 4-row K groups (SBO 512 B), 32-element N chunks one TMA box apart
              bh = smem_desc(b_hi + kk * 1024, BK * 128, 512, kLayoutSw128Base32);
              bl = smem_desc(b_lo + kk * 1024, BK * 128, 512, kLayoutSw128Base32);
            }
            umma_tf32(d_small, al, bh, idesc, first ? 0u : 1u);
            umma_tf32(d_small, ah, bl, idesc, 1u);
            umma_tf32(d_big, ah, bh, idesc, first ? 0u : 1u);
            first = false;
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[buf]);
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    float* stg = tr + q * 2 * 1024;
    uint32_t chunk = 0;
    int lt = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++lt) {
      const TileInfo ti = tile_info(p, t);
      const int buf = lt & 1;
      const uint32_t use = static_cast<uint32_t>(lt >> 1);
      if (!mbar_wait(&acc_full[buf], use & 1u, p.st, 15)) break;
      tc_fence_after();
      const bool has_k = ti.kb1 > ti.kb0;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(buf * 2 * BN);
      const int row0 = ti.mt * BM + q * 32;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        {
          float vs[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);         // hi.hi; lane = row, v[i] = column i
          tmem_ld_32x32b_x32(taddr + BN + c * 32, vs);   // cross terms
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] += vs[i];
        }
        // 32 x 32 staging tile in the TMA 128-byte swizzle: 16-byte chunk k of
        // row r sits at chunk k ^ (r % 8); double-buffered per warp
        float* sb = stg + (chunk & 1) * 1024;
        if (lane == 0) bulk_wait_read<1>();  // this buffer's previous store has read it
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 o = has_k ? make_float4(p.alpha * v[4 * k], p.alpha * v[4 * k + 1],
                                               p.alpha * v[4 * k + 2], p.alpha * v[4 * k + 3])
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(sb + lane * 32 + ((k ^ (lane & 7)) << 2)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < ti.M) {
          if (p.reduce_add)
            tma_reduce_add_3d(&tmC, sb, ti.nt * BN + c * 32, row0, ti.z);
          else
            tma_store_3d(&tmC, sb, ti.nt * BN + c * 32, row0, ti.z);
        }
        if (lane == 0) bulk_commit();
        ++chunk;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (lane == 0) bulk_wait_all();  // every store of this CTA has landed
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

EncodeTiledFn encode_fn_f32() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    tried = true;
  }
  return fn;
}

// fp32 3-D map {inner, outer, batch} with the given row and batch strides (elements).
bool make_map_f32(CUtensorMap* map, const float* base, int64_t inner, int64_t outer,
                  int64_t ld, int batch, int64_t bstride, uint32_t box_inner,
                  uint32_t box_outer, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn_f32();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                              static_cast<cuuint64_t>(batch)};
  const int64_t bs = batch > 1 ? bstride : ld * outer;
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 4, static_cast<cuuint64_t>(bs) * 4};
  const cuuint32_t box[3] = {box_inner, box_outer, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool ok16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

int launch_tc_sgemm(int M, int N, int K, float alpha, const float* A, int64_t lda,
                    const float* B, int64_t ldb, bool trans_b, float beta, float* C, int64_t ldc,
                    int mode, DeviceStatus* st, cudaStream_t stream, const GemmBatch& bt) {
  if (M <= 0 || N <= 0 || bt.count < 1) return PIQ_OK;
  if (mode == 1 && M != N) return PIQ_ERR_INVALID_ARG;
  if (bt.m_total > 0) {
    // A tensor map covers every entry with the same extent, so a short last
    // entry gets a launch of its own with exact extents: no load ever reaches
    // past the memory an entry owns.
    const int64_t last = bt.m_total - static_cast<int64_t>(bt.count - 1) * bt.m_step;
    GemmBatch full = bt;
    full.m_total = 0;
    full.k_follows_m = false;
    if (last >= M) {
      return launch_tc_sgemm(M, N, K, alpha, A, lda, B, ldb, trans_b, beta, C, ldc, mode, st,
                             stream, full);
    }
    if (!ok16(A) || !ok16(B) || !ok16(C) || (lda & 3) || (ldb & 3) || (ldc & 3) ||
        (bt.stride_a & 3) || (bt.stride_b & 3) || (bt.stride_c & 3) ||
        (beta != 0.f && beta != 1.f))
      return PIQ_ERR_INVALID_ARG;
    if (bt.count > 1) {
      full.count = bt.count - 1;
      const int rc = launch_tc_sgemm(M, N, K, alpha, A, lda, B, ldb, trans_b, beta, C, ldc,
                                     mode, st, stream, full);
      if (rc != PIQ_OK) return rc;
    }
    if (last <= 0) return PIQ_OK;
    const int64_t z = bt.count - 1;
    const int ml = static_cast<int>(last);
    return launch_tc_sgemm(ml, N, bt.k_follows_m ? ml : K, alpha, A + z * bt.stride_a, lda,
                           B + z * bt.stride_b, ldb, trans_b, beta, C + z * bt.stride_c, ldc,
                           mode, st, stream, GemmBatch());
  }
  // TMA: 16-byte aligned bases and row strides
  if (!ok16(A) || !ok16(B) || !ok16(C) || (lda & 3) || (ldb & 3) || (ldc & 3) ||
      (bt.count > 1 && ((bt.stride_a & 3) || (bt.stride_b & 3) || (bt.stride_c & 3))))
    return PIQ_ERR_INVALID_ARG;
  if (beta != 0.f && beta != 1.f) return PIQ_ERR_INVALID_ARG;  // store or reduce-add only
  DeviceInfo info;
  int rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  CUtensorMap ma, mb;
  if (!make_map_f32(&ma, A, K, M, lda, bt.count, bt.stride_a, BK, BM)) return PIQ_ERR_INVALID_ARG;
  const bool okb = trans_b ? make_map_f32(&mb, B, K, N, ldb, bt.count, bt.stride_b, BK, BN)
                           : make_map_f32(&mb, B, N, K, ldb, bt.count, bt.stride_b, 32, BK,
                                          CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  if (!okb) return PIQ_ERR_INVALID_ARG;
  CUtensorMap mc;
  if (!make_map_f32(&mc, C, N, M, ldc, bt.count, bt.stride_c, 32, 32)) return PIQ_ERR_INVALID_ARG;
  SgParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.alpha = alpha;
  p.beta = beta;
  p.C = C;
  p.ldc = ldc;
  p.mode = mode;
  p.trans_b = trans_b;
  p.m_tiles = static_cast<int>(ceil_div(M, BM));
  p.n_tiles = static_cast<int>(ceil_div(N, BN));
  p.tiles_per_z = mode == 1 ? p.m_tiles * (p.m_tiles + 1) / 2 : p.m_tiles * p.n_tiles;
  p.batch = bt.count;
  const int64_t total = static_cast<int64_t>(p.tiles_per_z) * bt.count;
  if (total > INT32_MAX) return PIQ_ERR_INVALID_ARG;
  p.num_tiles = static_cast<int>(total);
  p.stride_c = bt.stride_c;
  p.m_total = bt.m_total;
  p.m_step = bt.m_step;
  p.k_follows_m = bt.k_follows_m;
  p.reduce_add = beta != 0.f;
  p.st = st;

  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(tf32x3_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int grid = std::max(1, std::min(p.num_tiles, info.sm_count));
  note_launch();
  if (launch_pdl(tf32x3_gemm_kernel, dim3(grid), dim3(THREADS), SMEM_BYTES, stream, ma, mb, mc,
                 p) != cudaSuccess)
    return PIQ_ERR_CUDA;
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

static std::atomic<uint64_t> g_simt_fallbacks{0};

uint64_t simt_gemm_fallbacks() { return g_simt_fallbacks.load(); }

int launch_gemm_f32(int M, int N, int K, float alpha, const float* A, int64_t lda, const float* B,
                    int64_t ldb, bool trans_b, float beta, float* C, int64_t ldc, int mode,
                    DeviceStatus* st, cudaStream_t stream, const GemmBatch& bt) {
  const int rc = launch_tc_sgemm(M, N, K, alpha, A, lda, B, ldb, trans_b, beta, C, ldc, mode,
                                 st, stream, bt);
  if (rc != PIQ_ERR_INVALID_ARG) return rc;
  // an operand the tensor maps cannot describe (a base or row stride that is
  // not 16-byte aligned): counted, so callers can see which path ran
  g_simt_fallbacks.fetch_add(1);
  return launch_simt_gemm(M, N, K, alpha, A, lda, B, ldb, trans_b, beta, C, ldc, mode, st,
                          stream, bt);
}

}  // namespace piq
