// FP64-grade GEMM on the INT8 tensor cores (tcgen05 kind::i8), for the steps
// whose results decide rounding sites: the Cholesky factor of the damped
// Hessian and the GPTQ block updates.
//
// Why: the GPTQ listing of "GPTQ versus AWQ objectives" ("A strong answer")
// forms U = cholesky(inv(H)) and pushes every rounding error through it; at a
// 28672-column layer an FP32 factor (or FP32-accumulated updates) moves w/scale
// by ~1e-5, which flips several thousand rounding decisions against an FP64
// evaluation of the same loop.  B200 has ~37 TFLOP/s of FP64 but ~2.6 POP/s of
// INT8, so FP64-grade products are formed from exact integer ones.
//
// Method (splitting of floating-point operands into small integers, summed
// exactly in integer arithmetic; Ozaki et al., "Error-free transformations of
// matrix multiplication", and its integer-unit variants): every row of an
// operand is scaled by a power of two 2^e (e from frexp of the row's largest
// magnitude, so the row lies in (-1, 1)), and then written as
//     y = 2^-6 (q0 + 2^-7 (q1 + 2^-7 (q2 + ...)))
// with signed digits q_i in [-64, 64] (each step rounds to nearest, so the
// remainder stays in [-1/2, 1/2] and the next digit fits in 7 bits plus sign).
// s digits keep about 6 + 7 (s - 1) bits of every entry relative to its row's
// largest one.  For C = A B^T the integer products q_i(A) q_j(B) with the same
// weight 2^(-7 (i + j)) go to one int32 accumulator d = i + j in TMEM (exact:
// at most 64 * 64 * K * (d + 1) < 2^31 for K (d + 1) < 2^19); pairs with
// i + j >= s are dropped (their weight is below 2^(-7 s)).  The epilogue turns
// the s accumulators into one fp64 value by Horner's rule in powers of 2^-7,
// scales it by 2^(e_A(r) + e_B(c) - 12) and alpha, and adds it to (or stores
// it into) an fp64 C.  With s = 6 the relative error of each product sum is
// about 1e-12 of max|A_r| max|B_c| K, far below FP32 (6e-8).
//
// Layout: digits are stored K-major, q[i][row][kpad] int8 with kpad a multiple
// of 64 (zero padded), and the exponents e[row] int32.  Tiles: 128 rows of A x
// 48 rows of B, K in blocks of 64 bytes (64-byte swizzle); a pipeline stage
// holds all s digit tiles of A and of B for one k block, the B tiles one
// after another so that they read as a single K-major matrix of s * 48 rows.
// TMEM holds the s accumulators of a tile side by side (accumulator d at
// column 48 d), two tiles' worth (double-buffered).  Digit i of A times the
// stacked B digits 0 .. s-1-i is one MMA of N = 48 (s - i) whose output
// columns are exactly accumulators i .. s-1, i.e. pair (i, j) lands in
// accumulator i + j: s MMAs per 32-byte k step instead of s (s + 1) / 2 narrow
// ones, which halves the shared-memory operand reads that bound the tensor
// pipe at narrow N.
//
// Warp roles (320 threads): warp 0 lane 0 issues TMA loads; warp 1 lane 0
// issues the MMAs; warps 2..9 drain TMEM (warp w reads lanes 32 (w % 4) ..,
// two warps per lane quadrant, one per 24-column half of the tile), own 32
// half rows of C each, and add them into C with asynchronous bulk reduce-adds
// from shared memory.  Every wait is bounded; no multicast loads.
#include <cuda.h>

#include <algorithm>

#include "internal.h"

namespace piq {

namespace {

constexpr int BM = 128;
constexpr int BN = 48;                        // columns of C per tile
constexpr int BK = 64;                        // int8 digits = one 64-byte row
constexpr int A_TILE = BM * BK;               // 8 KB per digit
constexpr int B_TILE = BN * BK;               // 3 KB per digit
constexpr int EPI_WARPS = 8;                  // two per TMEM lane quadrant, one per half tile
constexpr int HALF = BN / 2;                  // columns of C per epilogue warp
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int MAX_SMEM = 227 * 1024;
constexpr int BUF_COLS = 256;                 // TMEM columns between the two accumulator sets
constexpr int STG_LD = HALF + 2;              // fp64 staging row stride (16-byte rows, 4-way banks)
constexpr int STG_WARP = 32 * STG_LD + HALF;  // doubles per epilogue warp: 32 rows + column scales
constexpr int STG_BYTES = EPI_WARPS * STG_WARP * 8;

struct OzParams {
  int M, N, K, s;
  int m_tiles, n_tiles, num_tiles;
  int stages;
  int stage_bytes;
  double alpha;
  int beta;             // 0: C = alpha A B^T; 1: C += alpha A B^T
  int lower;            // only entries c <= r (tiles touching the lower triangle)
  double* C;
  int64_t ldc;
  const int* ea;
  const int* eb;
  DeviceStatus* st;
};

// Column tiles of row tile m that reach the lower triangle: n BN <= 128 m + 127.
__host__ __device__ __forceinline__ int lower_cols(int m, int n_tiles) {
  return min(n_tiles, (BM * m + BM - 1) / BN + 1);
}

// Tiles in row tiles 0 .. m - 1 of a lower launch, in closed form.  With
// 128 x 48 tiles, row tile i = 3 a + b reaches column tile 8 a + {2, 5, 7}[b],
// so three consecutive rows hold 24 a + 17 tiles; rows from the first one whose
// count reaches n_tiles on hold n_tiles each.
static_assert(BM == 128 && BN == 48, "lower_prefix assumes 128 x 48 tiles");
__host__ __device__ __forceinline__ int64_t lower_prefix(int m, int n_tiles) {
  const int64_t x = static_cast<int64_t>(BN) * (n_tiles - 1) - (BM - 1);
  const int64_t m_full = x > 0 ? (x + BM - 1) / BM : 0;  // first row with n_tiles tiles
  const int k = static_cast<int>(m < m_full ? m : m_full);
  const int64_t a = k / 3;
  const int b = k - 3 * static_cast<int>(a);
  const int64_t part = b == 0 ? 0 : (b == 1 ? 8 * a + 3 : 16 * a + 9);
  return 12 * a * (a - 1) + 17 * a + part +
         (m > m_full ? m - m_full : 0) * static_cast<int64_t>(n_tiles);
}

// Tile t of the launch.  Tiles run in groups of RG row tiles: inside a group
// the column tiles are the outer loop, so that a wave of persistent CTAs works
// on a few column blocks of B for RG row blocks of A and B's digits are read
// from DRAM once per group rather than once per row tile (at N = 27648 and
// K = 1024 they are 141 MB, more than L2 keeps).  A lower launch finds its
// group by bisection on lower_prefix, walks the group's full columns the same
// way, then its staircase row by row.
constexpr int RG = 8;

__host__ __device__ __forceinline__ void tile_of(const OzParams& p, int t, int& mt, int& nt) {
  if (p.lower) {
    int lo = 0, hi = (p.m_tiles + RG - 1) / RG - 1;  // the last group g with prefix <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (lower_prefix(mid * RG, p.n_tiles) <= t)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int m0 = lo * RG;
    const int gs = min(RG, p.m_tiles - m0);
    int r = t - static_cast<int>(lower_prefix(m0, p.n_tiles));
    const int c0 = lower_cols(m0, p.n_tiles);  // columns every row of the group has
    if (r < gs * c0) {
      nt = r / gs;
      mt = m0 + r - nt * gs;
      return;
    }
    r -= gs * c0;
    for (int m = m0; m < m0 + gs; ++m) {
      const int extra = lower_cols(m, p.n_tiles) - c0;
      if (r < extra) {
        mt = m;
        nt = c0 + r;
        return;
      }
      r -= extra;
    }
    mt = nt = 0;
  } else {
    const int full = RG * p.n_tiles;  // tiles of a complete group
    const int m0 = (t / full) * RG;
    const int gs = min(RG, p.m_tiles - m0);
    const int r = t - m0 * p.n_tiles;
    nt = r / gs;
    mt = m0 + r - nt * gs;
  }
}

// Instruction descriptor: kind::i8, signed A and B, s32 accumulate, K-major
// A and B, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

constexpr uint32_t kLayoutSw64 = 4;  // smem descriptor: 64-byte swizzle

// 2^e for e well inside the normal range, from the exponent field.
__device__ __forceinline__ double pow2i(int e) {
  return __longlong_as_double(static_cast<long long>(1023 + e) << 52);
}

// S (digits per operand) is a template parameter so that the MMA issue loop
// unrolls into straight-line code with constant descriptors.
template <int S>
__global__ void __launch_bounds__(THREADS, 1)
    ozaki_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, OzParams p) {
  static_assert(S * BN <= 256 && S * BN <= BUF_COLS, "stacked digits exceed one MMA");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  double* stg_all = reinterpret_cast<double*>(smem + p.stages * p.stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.stages * p.stage_bytes + STG_BYTES);
  uint64_t* empty = full + p.stages;
  uint64_t* acc_full = empty + p.stages;  // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.K + BK - 1) / BK;
  pdl_wait();
  const bool skip = status_bad(p.st);

  if (skip) {
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_of(p, t, mt, nt);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int st = it % p.stages;
          const uint32_t ph = (it / p.stages) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, p.st, 41)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * p.stage_bytes;
          uint8_t* sb = sa + S * A_TILE;  // B digits stacked: one S*BN-row K-major matrix
          mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(p.stage_bytes));
          for (int i = 0; i < S; ++i) {
            tma_load_3d(sa + i * A_TILE, &tmA, &full[st], kb * BK, mt * BM, i);
            tma_load_3d(sb + i * B_TILE, &tmB, &full[st], kb * BK, nt * BN, i);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      // Digit i of A against B digits 0 .. S-1-i stacked (N = (S - i) BN) lands
      // in accumulators i .. S-1, i.e. pair (i, j) in accumulator i + j: one
      // MMA per A digit and 32-byte k step.
      uint32_t it = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++lt) {
        const int buf = lt & 1;
        const uint32_t use = static_cast<uint32_t>(lt >> 1);
        if (!mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, p.st, 42)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * BUF_COLS);
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int st = it % p.stages;
          const uint32_t ph = (it / p.stages) & 1u;
          if (!mbar_wait(&full[st], ph, p.st, 43)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + st * p.stage_bytes);
          const uint64_t ad0 = smem_desc(a0, 16, 512, kLayoutSw64);
          const uint64_t bd0 = smem_desc(a0 + S * A_TILE, 16, 512, kLayoutSw64);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
#pragma unroll
            for (int i = 0; i < S; ++i) {
              // digit 0 of A covers every accumulator: it starts the tile
              const uint32_t acc = (kb == 0 && kk == 0 && i == 0) ? 0u : 1u;
              umma_i8(d0 + static_cast<uint32_t>(i * BN),
                      ad0 + static_cast<uint64_t>(i * (A_TILE >> 4) + kk * 2),
                      bd0 + static_cast<uint64_t>(kk * 2), idesc_i8((S - i) * BN), acc);
            }
          }
          umma_commit(&empty[st]);
        }
        if (ok) umma_commit(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp: the left or right half of 32 rows of the tile (lane = row).
    // TMEM -> registers, Horner in powers of 2^-7, times 2^e_A(row) alpha 2^(e_B(col) - 12), into
    // the lane's row of the warp's staging block; the TMEM buffer goes back
    // to the MMA issuer; then one asynchronous bulk copy per row adds the row
    // segment into C in global memory (or stores it when beta = 0), so that
    // the read-modify-write of C happens at L2 without a round trip through
    // the SM.  A row whose segment is not 16-byte aligned or has an odd
    // length finishes with plain accesses.
    const int q = warp & 3;         // TMEM lanes 32 q .. 32 q + 31: rows of the tile
    const int h = (warp - 2) >> 2;  // columns h HALF .. h HALF + HALF - 1 of the tile
    double* stg = stg_all + (warp - 2) * STG_WARP;
    double* cs = stg + 32 * STG_LD;
    int lt = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++lt) {
      int mt, nt;
      tile_of(p, t, mt, nt);
      const int buf = lt & 1;
      const uint32_t use = static_cast<uint32_t>(lt >> 1);
      const int col0 = nt * BN + h * HALF;
      const int row = mt * BM + q * 32 + lane;
      if (!mbar_wait(&acc_full[buf], use & 1u, p.st, 44)) break;
      tc_fence_after();
      bulk_wait_read<0>();  // this lane's earlier bulk copies are done reading its row
      if (lane < HALF) {
        const int col = col0 + lane;
        cs[lane] = col < p.N ? p.alpha * pow2i(__ldg(p.eb + col) - 12) : 0.0;
      }
      __syncwarp();
      const double rsc = pow2i(row < p.M ? __ldg(p.ea + row) : 0);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(buf * BUF_COLS + h * HALF);
      double* srow = stg + lane * STG_LD;
#pragma unroll
      for (int c = 0; c < HALF / 8; ++c) {
        double v[8];
        float f[8];
        tmem_ld_32x32b_x8(taddr + static_cast<uint32_t>((S - 1) * BN + 8 * c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = static_cast<double>(__float_as_int(f[i]));
#pragma unroll
        for (int d = S - 2; d >= 0; --d) {
          tmem_ld_32x32b_x8(taddr + static_cast<uint32_t>(d * BN + 8 * c), f);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            v[i] = fma(v[i], 0.0078125, static_cast<double>(__float_as_int(f[i])));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) srow[8 * c + i] = (v[i] * rsc) * cs[8 * c + i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (row < p.M) {
        int ncol = min(HALF, p.N - col0);
        if (p.lower) ncol = min(ncol, row - col0 + 1);  // c <= r
        if (ncol > 0) {
          double* crow = p.C + static_cast<int64_t>(row) * p.ldc + col0;
          const int nbulk = (reinterpret_cast<uintptr_t>(crow) & 15u) == 0 ? (ncol & ~1) : 0;
          if (nbulk > 0) {
            fence_proxy_async_smem();
            if (p.beta)
              bulk_reduce_add_f64(crow, srow, static_cast<uint32_t>(nbulk * 8));
            else
              bulk_store_global(crow, srow, static_cast<uint32_t>(nbulk * 8));
            bulk_commit();
          }
          for (int c = nbulk; c < ncol; ++c) crow[c] = p.beta ? crow[c] + srow[c] : srow[c];
        }
      }
    }
    bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ----------------------------------------------------------------- digits
// Row r of the logical rows x K matrix: element (r, k) at src[r * rs + k * ks].
// One warp per row, lane l holding entries 4 l .. 4 l + 3 of each 128-entry
// chunk.  Rows of up to 128 CH entries are read once into registers (every
// load issued before any is used), their largest magnitude found by a warp
// reduction, and the s digits of every entry written from the registers
// (zeros for k in [K, kpad)); longer rows take two passes.
template <int S>
__device__ __forceinline__ void write_digits4(const double (&x)[4], double sc6, int8_t* q,
                                              int64_t plane, int64_t off) {
  double y[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) y[t] = x[t] * sc6;  // |y| < 64
#pragma unroll
  for (int i = 0; i < S; ++i) {
    uint32_t w = 0;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const double di = rint(y[t]);
      y[t] = (y[t] - di) * 128.0;
      w |= (static_cast<uint32_t>(static_cast<int>(di)) & 0xFFu) << (8 * t);
    }
    *reinterpret_cast<uint32_t*>(q + i * plane + off) = w;
  }
}

template <int S, int CH>
__global__ void slice_rows_kernel(const double* __restrict__ src, int64_t rs, int64_t ks,
                                  int64_t rows, int64_t K, int8_t* __restrict__ q, int64_t kpad,
                                  int* __restrict__ ex) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const double* row = src + r * rs;
  const int64_t plane = rows * kpad;
  const int64_t nch = (kpad + 127) / 128;
  double m = 0.0;
  double x[CH][4];
  if (nch <= CH) {
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int64_t k = 128 * c + 4 * lane + t;
        x[c][t] = (c < nch && k < K) ? row[k * ks] : 0.0;
      }
#pragma unroll
    for (int c = 0; c < CH; ++c)
#pragma unroll
      for (int t = 0; t < 4; ++t) m = fmax(m, fabs(x[c][t]));
  } else {
    for (int64_t k = lane; k < K; k += 32) m = fmax(m, fabs(row[k * ks]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  int e = 0;
  if (m > 0.0) frexp(m, &e);  // m = f 2^e with f in [0.5, 1)
  if (lane == 0) ex[r] = e;
  // 2^(6 - e) from its exponent field (row maxima stay far inside the normal range);
  // an all-zero row gets zero digits
  const double sc6 =
      m > 0.0 ? __longlong_as_double(static_cast<long long>(1023 + 6 - e) << 52) : 0.0;
  if (nch <= CH) {
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const int64_t k0 = 128 * c + 4 * lane;
      if (c < nch && k0 < kpad) write_digits4<S>(x[c], sc6, q, plane, r * kpad + k0);
    }
  } else {
    for (int64_t k0 = 4 * lane; k0 < kpad; k0 += 128) {
      double v[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) v[t] = (k0 + t < K) ? row[(k0 + t) * ks] : 0.0;
      write_digits4<S>(v, sc6, q, plane, r * kpad + k0);
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_i8() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    tried = true;
  }
  return fn;
}

// int8 digit planes [s][rows][kpad] as a 3-D map {kpad, rows, s}, box {64, box_rows, 1}.
bool make_digit_map(CUtensorMap* map, const DigitMat& d, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn_i8();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d.kpad), static_cast<cuuint64_t>(d.rows),
                              static_cast<cuuint64_t>(d.s)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d.kpad),
                                 static_cast<cuuint64_t>(d.plane ? d.plane : d.rows * d.kpad)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(d.q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int64_t digit_kpad(int64_t K) { return (K + BK - 1) / BK * BK; }

int launch_slice(const double* src, int64_t rs, int64_t ks, int64_t rows, int64_t K, int s,
                 DigitMat* out, cudaStream_t stream) {
  if (rows < 1 || K < 1 || s < 1 || s > kMaxDigits) return PIQ_ERR_INVALID_ARG;
  if (out->kpad != digit_kpad(K) || out->s != s || out->rows != rows) return PIQ_ERR_INVALID_ARG;
  if (out->plane != 0 && out->plane != rows * out->kpad) return PIQ_ERR_INVALID_ARG;  // no views
  const int64_t threads = rows * 32;
  const unsigned grid = static_cast<unsigned>(ceil_div(threads, 256));
  void (*kern)(const double*, int64_t, int64_t, int64_t, int64_t, int8_t*, int64_t, int*) = nullptr;
  const bool short_row = out->kpad <= 128;
  switch (s) {
    case 1: kern = short_row ? slice_rows_kernel<1, 1> : slice_rows_kernel<1, 8>; break;
    case 2: kern = short_row ? slice_rows_kernel<2, 1> : slice_rows_kernel<2, 8>; break;
    case 3: kern = short_row ? slice_rows_kernel<3, 1> : slice_rows_kernel<3, 8>; break;
    case 4: kern = short_row ? slice_rows_kernel<4, 1> : slice_rows_kernel<4, 8>; break;
    case 5: kern = short_row ? slice_rows_kernel<5, 1> : slice_rows_kernel<5, 8>; break;
    case 6: kern = short_row ? slice_rows_kernel<6, 1> : slice_rows_kernel<6, 8>; break;
    case 7: kern = short_row ? slice_rows_kernel<7, 1> : slice_rows_kernel<7, 8>; break;
    default: break;
  }
  if (kern == nullptr) return PIQ_ERR_INVALID_ARG;
  note_launch();
  kern<<<grid, 256, 0, stream>>>(src, rs, ks, rows, K, out->q, out->kpad, out->ex);
  return launch_ok("digit split launch") ? PIQ_OK : PIQ_ERR_CUDA;
}

int launch_ozaki_gemm(int64_t M, int64_t N, const DigitMat& A, const DigitMat& B, double alpha,
                      int beta, int lower, double* C, int64_t ldc, DeviceStatus* st,
                      cudaStream_t stream, int max_ctas) {
  if (M <= 0 || N <= 0) return PIQ_OK;
  if (A.s != B.s || A.kpad != B.kpad || A.rows < M || B.rows < N || A.s < 3 || A.s > 5)
    return PIQ_ERR_INVALID_ARG;
  if (A.kpad * (A.s + 1) >= (int64_t)1 << 19) return PIQ_ERR_INVALID_ARG;  // int32 exactness
  if (M > INT32_MAX || N > INT32_MAX) return PIQ_ERR_INVALID_ARG;
  DeviceInfo info;
  int rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  CUtensorMap ma, mb;
  if (!make_digit_map(&ma, A, BM) || !make_digit_map(&mb, B, BN))
    return PIQ_ERR_INVALID_ARG;
  OzParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(A.kpad);
  p.s = A.s;
  p.m_tiles = static_cast<int>(ceil_div(M, BM));
  p.n_tiles = static_cast<int>(ceil_div(N, BN));
  if (lower) {
    const int64_t tot = lower_prefix(p.m_tiles, p.n_tiles);
    if (tot > INT32_MAX) return PIQ_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tot);
  } else {
    const int64_t tot = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
    if (tot > INT32_MAX) return PIQ_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tot);
  }
  p.stage_bytes = p.s * (A_TILE + B_TILE);
  p.stages = std::min(4, (MAX_SMEM - 1024 - 256 - STG_BYTES) / p.stage_bytes);
  if (p.stages < 2) return PIQ_ERR_INVALID_ARG;
  p.alpha = alpha;
  p.beta = beta ? 1 : 0;
  p.lower = lower ? 1 : 0;
  p.C = C;
  p.ldc = ldc;
  p.ea = A.ex;
  p.eb = B.ex;
  p.st = st;
  // the pipeline stages, the epilogue's staging blocks and the barriers; more
  // than half an SM's shared memory, so that two CTAs that each hold all 512
  // TMEM columns never share an SM
  const int smem = std::max(p.stages * p.stage_bytes + STG_BYTES + 1024 + 256, 120 * 1024);
  void (*kern)(CUtensorMap, CUtensorMap, OzParams) = nullptr;
  switch (p.s) {
    case 3: kern = ozaki_gemm_kernel<3>; break;
    case 4: kern = ozaki_gemm_kernel<4>; break;
    case 5: kern = ozaki_gemm_kernel<5>; break;
    default: return PIQ_ERR_INVALID_ARG;
  }
  static bool attr_set[64][8] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  if (dev < 64 && !attr_set[dev][p.s]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MAX_SMEM) !=
        cudaSuccess)
      return PIQ_ERR_CUDA;
    attr_set[dev][p.s] = true;
  }
  // max_ctas > 0 leaves SMs free for work on another stream
  const int ctas = max_ctas > 0 ? std::min(max_ctas, info.sm_count) : info.sm_count;
  const int grid = std::max(1, std::min(p.num_tiles, ctas));
  // algorithmic work: 2 K operations per computed entry of C and digit pair
  double entries = static_cast<double>(M) * static_cast<double>(N);
  if (lower)
    entries = (N <= M) ? static_cast<double>(N) * (N + 1) / 2 + static_cast<double>(M - N) * N
                       : static_cast<double>(M) * (M + 1) / 2;
  const int slot = gemm_timing_begin(stream);
  note_launch();
  if (launch_pdl(kern, dim3(grid), dim3(THREADS), static_cast<size_t>(smem), stream, ma, mb, p) !=
      cudaSuccess)
    return PIQ_ERR_CUDA;
  gemm_timing_end(slot, stream, 2.0 * entries * static_cast<double>(p.K) * p.s * (p.s + 1) / 2);
  return launch_ok() ? PIQ_OK : PIQ_ERR_CUDA;
}

}  // namespace piq

// The order in which the digit GEMM's persistent CTAs take their tiles (tile
// t of a launch is taken by CTA t mod grid), for tests and tools.
extern "C" int64_t piq_gemm_tile_order(int m_tiles, int n_tiles, int lower, int64_t count,
                                       int* mt, int* nt) {
  using namespace piq;
  if (m_tiles < 1 || n_tiles < 1) return PIQ_ERR_INVALID_ARG;
  const int64_t total = lower ? lower_prefix(m_tiles, n_tiles)
                              : static_cast<int64_t>(m_tiles) * n_tiles;
  if (total > INT32_MAX) return PIQ_ERR_INVALID_ARG;
  if (mt == nullptr || nt == nullptr) return total;
  if (count < total) return PIQ_ERR_INVALID_ARG;
  OzParams p{};
  p.m_tiles = m_tiles;
  p.n_tiles = n_tiles;
  p.num_tiles = static_cast<int>(total);
  p.lower = lower ? 1 : 0;
  for (int t = 0; t < p.num_tiles; ++t) tile_of(p, t, mt[t], nt[t]);
  return total;
}
