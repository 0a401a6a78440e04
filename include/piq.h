/*
 * piq.h - C ABI of the B200 (sm_100a) layer-wise weight quantizer.
 *
 * One linear layer W[out, in] (fp32, row-major) and calibration inputs
 * X[n, in] (bfloat16 bit patterns, row-major) go in; packed INT4/INT3 codes,
 * FP16 group scales and the layer output error come out.  Two methods:
 *
 *   GPTQ  - "GPTQ versus AWQ objectives" (inferenceinterviews.com), section
 *           "A strong answer": proxy Hessian H = X^T X, damping by
 *           damp * mean(diag H), the upper Cholesky factor U of H^-1, then a
 *           column-by-column symmetric round-to-nearest with a per-row group
 *           scale max|W[:, j:j+g]| / qmax taken at each group start, codes
 *           clipped to [-qmax-1, qmax] (qmax = 2^(bits-1) - 1), and each
 *           rounding error (W[:, j] - Q[:, j]) / U[j, j] pushed onto the
 *           columns not yet quantized; updates are batched over column blocks
 *           so the trailing update is a GEMM.  Section "What interviewers probe
 *           next": act-order (columns by decreasing diag H, which needs a group
 *           index per column) and the 1% damping term.
 *   AWQ   - same page and section (AWQ paragraph): s_j = mean_n |x_nj|^alpha,
 *           W diag(s) rounded to nearest, one alpha per layer chosen by grid
 *           search on the calibration output error ||X W^T - X What^T||^2.
 *
 * Two widenings of GPTQ: AWQ's scaling first and GPTQ's rounding after (the
 * same page's serving decision list: the two compose; awq_gptq_quantize_layer),
 * and a scale plus a zero-point per group (the uplatz.com report, GPTQ's key
 * parameters, Group Size; gptq_quantize_layer_asym).
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers of the current device;
 *    "host" pointers are ordinary host memory.  The caller owns every buffer.
 *    The library never allocates device memory, never frees, and never writes
 *    W or X.  Scratch memory comes from the caller's `workspace` (device, at
 *    least 256-byte aligned), sized by the matching *_workspace_bytes query.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it.  Entry points that return host scalars synchronize the
 *    stream once before returning.
 *  - Device pointers must be 16-byte aligned; `in` must be a multiple of 8.
 *  - Return value: PIQ_OK (0) or a negative PIQ_ERR_* code.  On error the
 *    contents of the outputs are unspecified.
 *  - Packed format (this library's own; the pages fix only "the same INT4 plus
 *    group scales"): code c of memory-order column k is stored as
 *    u = c + 2^(bits-1) in bits [4*(k%8), 4*(k%8)+4) of uint32 word k/8 of its
 *    row (qweight is [out, in/8]).  scales is [out, ceil(in/g)] IEEE fp16 bit
 *    patterns, round-to-nearest-even of the fp32 scale the quantizer used.
 *    The dequantized weight is code * scale[row, group(k)] (GPTQ, RTN) and
 *    code * scale[row, group(k)] / s[k] (AWQ).  With a zero-point per group
 *    (gptq_quantize_layer_asym) the nibble holds u = c + zero[row, group(k)]
 *    instead, zeros being uint8 [out, ceil(in/g)].
 */
#ifndef PIQ_H_
#define PIQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum piq_status {
  PIQ_OK = 0,
  PIQ_ERR_INVALID_ARG = -1,          /* a size, pointer, alignment or parameter is invalid */
  PIQ_ERR_WORKSPACE_TOO_SMALL = -2,  /* ws_bytes below the matching *_workspace_bytes */
  PIQ_ERR_NOT_PD = -3,               /* damped H has a non-positive Cholesky pivot */
  PIQ_ERR_CUDA = -4,                 /* a CUDA runtime call or launch failed */
  PIQ_ERR_TIMEOUT = -5,              /* a bounded in-kernel wait gave up */
  PIQ_ERR_UNSUPPORTED_DEVICE = -6    /* the current device is not sm_100 */
};

/* Static text for a status code (never NULL). */
const char* piq_status_string(int status);

/* Bytes of the fp32 proxy Hessian of a layer with `in` inputs: in * in * 4.
 * ("GPTQ versus AWQ objectives", sizing block under "A strong answer":
 * H is in x in, FP32; 8,192^2 x 4 B = 268 MB, 28,672^2 x 4 B = 3.29 GB.) */
int piq_hessian_bytes(int64_t in, size_t* bytes);

/* H = X^T X  (or H += X^T X when accumulate != 0), the listing's proxy Hessian.
 *   X  device bf16 [n, in] row-major, read-only.
 *   H  device fp32 [in, in] row-major.  Every element on or above the diagonal
 *      is written (H[i][j], j >= i); elements below the diagonal are
 *      unspecified.  BF16 products, FP32 accumulation on the tensor cores in
 *      chunks of 1024 samples; the chunks are added into H in sample order
 *      (FP32), so the result is deterministic.
 * n >= 1, in >= 8, in % 8 == 0; X and H 16-byte aligned (else
 * PIQ_ERR_INVALID_ARG). */
int piq_hessian(const uint16_t* X, int64_t n, int64_t in, float* H, int accumulate,
                void* stream);

/* Damping and upper factor ("A strong answer" listing; "What interviewers probe
 * next", damping):  H_p = H[perm][:, perm] (identity when perm == NULL),
 * lambda = damp * mean(diag H_p),  U upper triangular with
 * (H_p + lambda I)^-1 = U^T U.
 *   H     device fp32 [in, in]; only the upper triangle (j >= i) is read.
 *   perm  device int32 [in] or NULL: perm[p] = memory column quantized at p.
 *   U     device fp32 [in, in]; upper triangle written, strict lower set to 0.
 *   lambda_out  host, may be NULL.
 * Returns PIQ_ERR_NOT_PD if a Cholesky pivot is not positive (e.g. X == 0). */
int piq_upper_factor_workspace_bytes(int64_t in, size_t* bytes);
int piq_upper_factor(const float* H, int64_t in, float damp, const int32_t* perm, float* U,
                     double* lambda_out, void* workspace, size_t ws_bytes, void* stream);

/* The column sweep alone, given U: GPTQ's rounding with error feedback on
 * weights already in quantization order ("A strong answer" listing, loop body;
 * the block-batched form of the remark after it).
 *   Wp      device fp32 [out, in], read-only (copied into the workspace).
 *   U       device fp32 [in, in], upper triangle read.
 *   codes   device int8 [out, in]: signed codes in quantization order.
 *   qscale  device fp32 [out, ceil(in/g)]: group scales in quantization order.
 * bits in {2,3,4}; g >= 1. */
int piq_gptq_sweep_workspace_bytes(int64_t out, int64_t in, size_t* bytes);
int piq_gptq_sweep(const float* Wp, int64_t out, int64_t in, const float* U, int bits, int g,
                   int8_t* codes, float* qscale, void* workspace, size_t ws_bytes,
                   void* stream);

/* Full GPTQ of one layer.
 *   W        device fp32 [out, in], read-only.
 *   X        device bf16 [n, in], read-only.
 *   bits     2, 3 or 4;  g >= 1 (g >= in: one group per row);  damp >= 0.
 *   act_order  0: natural column order; 1: decreasing diag(X^T X), ties by index.
 *   qweight  device uint32 [out, in/8], memory column order (see format above).
 *   scales   device fp16 [out, ceil(in/g)]; group p/g holds quantization
 *            positions [p, p+g) (memory order when act_order == 0).
 *   perm     device int32 [in] or NULL: memory column quantized at position p.
 *   g_idx    device int32 [in] or NULL: group of each memory-order column.
 *   out_err  host double, may be NULL: ||X W^T - X What^T||_F^2 with
 *            What = code * fp16(scale) (the layer a user reconstructs),
 *            evaluated as sum_r D_r H D_r^T (D = W - What in fp32) from the H
 *            of the first step: the same quantity, without a second pass over X.
 * Runs every step on the GPU: H (tensor cores), act-order, damping, the
 * blocked Cholesky factor R of the damped H (H_d = R R^T, so U = inv(R); FP64,
 * its products on the INT8 tensor cores with FP64 accumulation), the per-block
 * sweep in FP64 with the block updates on the same tensor-core path, packing,
 * output error.  The sweep uses the exact identity W0 - Q = U^T err (W0 the
 * weights before any update, Q = code * scale): it carries
 * acc = (W0 - Q) R to later columns and reads the current weights of a block
 * G as W0_G + acc_G inv(R_GG), the listing's arithmetic without forming U.
 * Synchronizes `stream` once at the end.
 * Workspace: piq_gptq_workspace_bytes with the same out, in, n, g and
 * act_order (the column blocks of the sweep depend on g). */
int piq_gptq_workspace_bytes(int64_t out, int64_t in, int64_t n, int g, int act_order,
                             size_t* bytes);
int gptq_quantize_layer(const float* W, int64_t out, int64_t in, const uint16_t* X, int64_t n,
                        int bits, int g, float damp, int act_order, uint32_t* qweight,
                        uint16_t* scales, int32_t* perm, int32_t* g_idx, double* out_err,
                        void* workspace, size_t ws_bytes, void* stream);

/* One layer split over several GPUs, in two calls around one exchange.
 * ("GPTQ versus AWQ objectives", sizing block under "A strong answer": H is an
 * in x in FP32 sum over the calibration samples, and one layer at a time fits
 * one GPU.  The sum splits over the samples; given H, the rows of W are
 * independent problems: the listing's updates never mix rows.)
 *
 * piq_layer_statistics: the statistics of one shard of the calibration samples.
 *   X      device bf16 [n, in] row-major (this shard's samples), read-only.
 *   H      device fp64 [in, in] row-major: on and above the diagonal, X^T X of
 *          this shard with FP64-grade sums (the same kernel as the layer call);
 *          below it, unspecified.  Summing the shards' H (an all-reduce of
 *          in * in doubles) gives the layer's H.
 *   sumsq  device fp64 [in] or NULL: sum_n x_nj^2 in exact FP64 sums, the
 *          act-order key; shards add up like H.
 *   Workspace: piq_layer_statistics_workspace_bytes.  Synchronizes once.
 *
 * gptq_quantize_rows_from_h: GPTQ of some rows of W given the layer's H.
 *   W      device fp32 [out, in]: these rows (any subset of the layer's rows).
 *   H      device fp64 [in, in], read-only: the upper triangle of the layer's
 *          X^T X (e.g. the all-reduced piq_layer_statistics outputs).
 *   sumsq  device fp64 [in]: the act-order key; required when act_order != 0.
 *   zeros  device uint8 [out, ceil(in/g)] or NULL: with it, a scale and a
 *          zero-point per group as in gptq_quantize_layer_asym.
 *   The other arguments and outputs are gptq_quantize_layer's, for these rows;
 *   out_err is these rows' share of ||X W^T - X What^T||^2 (the shares add up
 *   to the layer's).  Every rank computes the same damping, factor and perm.
 *   Workspace: piq_gptq_from_h_workspace_bytes.  Synchronizes once. */
int piq_layer_statistics_workspace_bytes(int64_t n, int64_t in, size_t* bytes);
int piq_layer_statistics(const uint16_t* X, int64_t n, int64_t in, double* H, double* sumsq,
                         void* workspace, size_t ws_bytes, void* stream);
int piq_gptq_from_h_workspace_bytes(int64_t out, int64_t in, int g, size_t* bytes);
int gptq_quantize_rows_from_h(const float* W, int64_t out, int64_t in, const double* H,
                              const double* sumsq, int bits, int g, float damp, int act_order,
                              uint32_t* qweight, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                              int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                              void* stream);

/* GPTQ with a scale and a zero-point per group (the uplatz.com report, GPTQ's
 * key parameters, Group Size).  The pages give no formula; the quantizer is
 * min/max affine rounding of the group's current weights over a range widened
 * to hold 0, taken at each group start like the symmetric scale:
 *   lo = min(0, min w), hi = max(0, max w),  scale = (hi - lo) / (2^bits - 1),
 *   zero = rint(-lo / scale)  (0 <= zero <= 2^bits - 1; 0 when scale is 0),
 *   u = clip(rint(w / scale) + zero, 0, 2^bits - 1),  What = (u - zero) * scale.
 *   qweight  as gptq_quantize_layer, but nibble = u (the stored code itself).
 *   zeros    device uint8 [out, ceil(in/g)], required: the zero-points, groups
 *            in quantization order like scales.
 *   out_err  What = (u - zero) * fp16(scale).
 * Workspace: piq_gptq_workspace_bytes.  Everything else as gptq_quantize_layer
 * (the error feedback, blocking, act-order and factor are unchanged). */
int gptq_quantize_layer_asym(const float* W, int64_t out, int64_t in, const uint16_t* X,
                             int64_t n, int bits, int g, float damp, int act_order,
                             uint32_t* qweight, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                             int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                             void* stream);

/* AWQ scale search of one layer.
 *   alpha_grid     host float [n_alpha], 1 <= n_alpha <= 64 (e.g. k/20, k = 0..19).
 *   best_alpha     host float, may be NULL: the grid value with the smallest
 *                  error (first one on a tie).
 *   s              device fp32 [in]: s_j = mean|x_j|^best_alpha (1 where the
 *                  mean is 0).  The caller folds 1/s into the previous op.
 *   qweight/scales as GPTQ; they quantize W' = W diag(s), so the layer's
 *                  weight is code * scale / s_j.
 *   err_per_alpha  host double [n_alpha], may be NULL:
 *                  ||X W^T - X What_alpha^T||^2 with What = code * scale / s
 *                  (full-precision scales, the search objective).
 * Synchronizes `stream` once at the end. */
int piq_awq_workspace_bytes(int64_t out, int64_t in, int64_t n, int n_alpha, size_t* bytes);
int awq_search_layer(const float* W, int64_t out, int64_t in, const uint16_t* X, int64_t n,
                     int bits, int g, const float* alpha_grid, int n_alpha, float* best_alpha,
                     float* s, uint32_t* qweight, uint16_t* scales, double* err_per_alpha,
                     void* workspace, size_t ws_bytes, void* stream);

/* AWQ's scaling first, GPTQ's rounding after ("GPTQ versus AWQ objectives",
 * the serving decision list: at 3 bits or similarly aggressive targets the two
 * compose; uplatz.com report, section 3.2: y = (W s)(X / s) is the same layer).
 * GPTQ, exactly as gptq_quantize_layer, of the layer W' = W diag(s) with
 * calibration inputs X' = X diag(1/s):
 *   H' = diag(1/s) X^T X diag(1/s) (X is not rescaled or re-rounded: H is
 *   built from X and scaled in FP64), act-order by decreasing diag(H'),
 *   damping and factor of H', the sweep over W diag(s) (fp32 products).
 *   s_ch       device fp32 [in], 16-byte aligned, every s_j finite and > 0
 *              (typically the s awq_search_layer returned).  A bad s_j is found
 *              on the device: PIQ_ERR_INVALID_ARG.  Read only.
 *   qweight/scales quantize W' (as awq_search_layer's do), so the layer's
 *              weight is code * scale / s_j.
 *   perm/g_idx as gptq_quantize_layer (perm: order of the scaled layer).
 *   out_err    host double, may be NULL:
 *              ||X W^T - X What^T||^2, What = code * fp16(scale) / s_j, taken
 *              through H' as sum_r D'_r H' D'_r^T with D' = W' - code * fp16(scale)
 *              (X' D'^T = X (W - What)^T).
 * Workspace: piq_gptq_workspace_bytes(out, in, n, act_order).  Other
 * arguments, layout, errors and synchronization as gptq_quantize_layer. */
int awq_gptq_quantize_layer(const float* W, int64_t out, int64_t in, const uint16_t* X,
                            int64_t n, const float* s_ch, int bits, int g, float damp,
                            int act_order, uint32_t* qweight, uint16_t* scales, int32_t* perm,
                            int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                            void* stream);

/* Plain group round-to-nearest (the "round-to-nearest" column of the toy table
 * in "GPTQ versus AWQ objectives"): every scale from the original weights, no
 * error feedback.  Same outputs and format as GPTQ with natural order.
 * Enqueues only; does not synchronize. */
int piq_rtn_workspace_bytes(int64_t out, int64_t in, size_t* bytes);
int piq_rtn_quantize_layer(const float* W, int64_t out, int64_t in, int bits, int g,
                           uint32_t* qweight, uint16_t* scales, void* workspace,
                           size_t ws_bytes, void* stream);

/* Output error of a packed layer on inputs X (the shared objective, "How to
 * approach it"; e.g. a held-out or shifted X'):
 *   ||X W^T - X What^T||_F^2,  What[r, k] = code * fp16(scale[r, grp(k)]) / s[k]
 * grp(k) = g_idx[k] (or k / g when g_idx == NULL); s == NULL means s = 1;
 * code = u - zeros[r, grp(k)] (uint8 [out, ceil(in/g)], asymmetric groups) or
 * u - 2^(bits-1) when zeros == NULL.
 * Two exact routes, picked from (out, in, n) alone so the workspace size is
 * fixed by them: directly, a BF16 tensor-core product X D^T (D = W - What
 * rounded to bf16) squared and summed; or, when n is large against out and in
 * (n in + 6 out in < 2 n out), through H = X^T X as sum_r D_r H D_r^T with D
 * in fp32 (FP32-accurate tensor-core GEMM).
 * All pointers device except out_err (host).  Synchronizes `stream`. */
int piq_output_error_workspace_bytes(int64_t out, int64_t in, int64_t n, size_t* bytes);
int piq_layer_output_error(const float* W, int64_t out, int64_t in, const uint32_t* qweight,
                           const uint16_t* scales, const uint8_t* zeros, const int32_t* g_idx,
                           const float* s, int bits, int g, const uint16_t* X, int64_t n,
                           double* out_err, void* workspace, size_t ws_bytes, void* stream);

/* Per-phase timing (diagnostics).  When enabled, gptq_quantize_layer and
 * awq_search_layer record CUDA events around their phases; the times of the
 * last such call are read back with piq_last_phase_times (milliseconds, in the
 * order of piq_phase_name(0..n-1)).  Host-side state, per process. */
int piq_set_timing(int enable);
int piq_last_phase_times(double* ms, int max_phases, int* n_phases);
const char* piq_phase_name(int i);
/* With timing on, the same call also records an event pair around every launch
 * of the INT8 digit GEMM (the FP64-grade products of the factor and the sweep):
 * *ms = their summed device time, *int8_ops = their algorithmic INT8 operations
 * (2 K per computed entry of C per digit pair, K padded to 64), *launches = the
 * number of launches.  Any pointer may be NULL.  Host-side state, per process. */
int piq_last_gemm_stats(double* ms, double* int8_ops, int* launches);

/* The tile order of the INT8 digit GEMM (host only, no device work): tiles are
 * 128 rows of C by 48 columns; a launch with m_tiles x n_tiles tiles (only the
 * tiles that reach the lower triangle when lower != 0: column tile n of row
 * tile m with 48 n <= 128 m + 127) takes them in groups of eight row tiles,
 * column tiles outer inside a group, then, for lower launches, each group's
 * remaining tiles row by row; persistent CTA c takes tiles c, c + grid, ...
 * Returns the launch's tile count, or a negative status (m_tiles or n_tiles
 * < 1, more than 2^31 - 1 tiles).  With mt and nt non-NULL (host int arrays of
 * `count` >= that many entries) tile t's row and column tile are written to
 * mt[t] and nt[t]; a smaller count is PIQ_ERR_INVALID_ARG. */
int64_t piq_gemm_tile_order(int m_tiles, int n_tiles, int lower, int64_t count, int* mt, int* nt);

/* Number of kernels this library has launched in this process (all devices);
 * a monotone diagnostic counter. */
uint64_t piq_kernel_launches(void);

/* Number of FP32-accurate GEMMs (the factor's panel updates and the sweep's
 * trailing updates) that ran on the SIMT FP32 kernel instead of the tensor
 * cores because an operand's base or row stride was not 16-byte aligned, as a
 * tensor-memory-accelerator copy requires.  Process-wide, monotone; both paths
 * give FP32-accurate results, the SIMT one more slowly. */
uint64_t piq_simt_gemm_fallbacks(void);

/* The last CUDA runtime error this library saw, as "<error name> in <where>"
 * ("" if none): what lies behind a PIQ_ERR_CUDA return (a launch the runtime
 * refused, or a kernel that failed, found when the call synchronized).
 * Host-side, per process; static storage, overwritten by the next error. */
const char* piq_last_cuda_error(void);

/* Self-test of the bounded device waits (no counterpart on the source pages:
 * part of this library's failure detection).  Every in-kernel wait of the
 * library gives up after a time limit (2 s in the compute calls), records
 * PIQ_ERR_TIMEOUT in the call's status word and lets its kernel return, so a
 * lost producer never hangs the GPU.  This call launches one block that waits,
 * through the same code, on a barrier nothing ever completes, with the limit
 * set to wait_ns; it returns PIQ_ERR_TIMEOUT (and the wait's site number in
 * *where_out, host, may be NULL) and leaves the context usable.
 *   wait_ns    1e3 .. 1e10 (else PIQ_ERR_INVALID_ARG)
 *   workspace  device, >= 256 bytes, 256-byte aligned (the status word)
 *   Synchronizes `stream` once.
 *
 * Host-side fault injection, for testing callers' error handling: with the
 * environment variable PIQ_FAULT set to "notpd", "timeout" or "oom", every
 * compute entry point (all but this one) returns PIQ_ERR_NOT_PD,
 * PIQ_ERR_TIMEOUT or PIQ_ERR_CUDA (reported by piq_last_cuda_error as an
 * injected cudaErrorMemoryAllocation) after checking its arguments and before
 * any device work.  Read at every call; unset or any other value: no effect. */
int piq_wait_selftest(uint64_t wait_ns, int* where_out, void* workspace, size_t ws_bytes,
                      void* stream);

/* piq_upper_factor without a caller workspace.  (The source pages have no
 * counterpart: this is a deployment variant of the damping + upper-factor step
 * above, same arguments minus the workspace, same results.)
 *
 * For callers that must not allocate device memory: code that runs inside
 * another framework's hook or plugin, where every device byte belongs to a
 * pool that framework owns, and callers that cannot afford cudaMalloc's
 * implicit device-wide synchronisation.  The scratch lives instead in a fixed
 * region inside this library (a file-scope __device__ array of about 2.4 MB
 * that every GPU which loads the library keeps until the process exits).
 *   - in <= PIQ_NOALLOC_MAX_IN (512); a larger in returns PIQ_ERR_INVALID_ARG
 *     and does nothing.  The call itself allocates and frees nothing.
 *   - The region is created by the CUDA driver when it loads this library's
 *     code onto a device.  With lazy module loading (CUDA's default) that
 *     happens at the first use on the device, which may be this entry's first
 *     call; a caller that must see no allocation at call time makes one
 *     warm-up call at initialisation (or sets CUDA_MODULE_LOADING=EAGER).
 *   - The first call on a device also looks up the region's device address
 *     for that device (cudaGetSymbolAddress, with that device current); make
 *     that first call before capturing any stream.
 *   - Errors: PIQ_ERR_INVALID_ARG for bad arguments, PIQ_ERR_NOT_PD as for
 *     piq_upper_factor, PIQ_ERR_CUDA for a failed runtime call (its name is
 *     then reported by piq_last_cuda_error).
 *   - All calls on a device share the one region, which keeps the last call's
 *     contents (the status word is cleared on every call).  Calls that overlap
 *     on the GPU (different streams or threads) race on it: serialise them.
 *   - Synchronizes `stream` once, like piq_upper_factor. */
#define PIQ_NOALLOC_MAX_IN 512
int piq_upper_factor_noalloc(const float* H, int64_t in, float damp, const int32_t* perm,
                             float* U, double* lambda_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PIQ_H_ */
