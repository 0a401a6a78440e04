// C-ABI entry points (include/piq.h): argument checks, workspace carving and
// the order of the steps.  Every step of the path runs in this library's
// kernels on the caller's stream; the host only launches and, at the end,
// reads back the status word and the host scalars.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace piq {

// ------------------------------------------------------------------ devices
int device_info(DeviceInfo* out) {
  static DeviceInfo cache[64];
  static bool have[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PIQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 64) return PIQ_ERR_CUDA;
  if (!have[dev]) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return PIQ_ERR_CUDA;
    cache[dev].sm_count = prop.multiProcessorCount;
    cache[dev].major = prop.major;
    cache[dev].minor = prop.minor;
    have[dev] = true;
  }
  *out = cache[dev];
  // the library holds sm_100a code only: compute capability 10.0 exactly
  return (cache[dev].major == 10 && cache[dev].minor == 0) ? PIQ_OK : PIQ_ERR_UNSUPPORTED_DEVICE;
}

static std::atomic<uint64_t> g_launches{0};
void note_launch(int count) { g_launches.fetch_add(static_cast<uint64_t>(count)); }

static std::mutex g_err_mu;
static char g_err_text[160] = "";
void note_cuda_error(cudaError_t e, const char* where) {
  std::lock_guard<std::mutex> lock(g_err_mu);
  snprintf(g_err_text, sizeof(g_err_text), "%s in %s", cudaGetErrorName(e), where);
}

int injected_fault() {
  const char* f = std::getenv("PIQ_FAULT");
  if (f == nullptr || *f == 0) return PIQ_OK;
  if (std::strcmp(f, "notpd") == 0) return PIQ_ERR_NOT_PD;
  if (std::strcmp(f, "timeout") == 0) return PIQ_ERR_TIMEOUT;
  if (std::strcmp(f, "oom") == 0) {
    note_cuda_error(cudaErrorMemoryAllocation, "PIQ_FAULT=oom (injected)");
    return PIQ_ERR_CUDA;
  }
  return PIQ_OK;
}

int cuda_rc(cudaError_t e) {
  if (e != cudaSuccess) note_cuda_error(e, "runtime call");
  return e == cudaSuccess ? PIQ_OK : PIQ_ERR_CUDA;
}

// Read the status word (and optional extra device bytes) after synchronizing.
int finish_call(DeviceStatus* st, cudaStream_t stream, DeviceStatus* host_st) {
  DeviceStatus tmp;
  cudaError_t e = cudaMemcpyAsync(&tmp, st, sizeof(DeviceStatus), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    note_cuda_error(e, "stream synchronization (a kernel of this call failed)");
    return PIQ_ERR_CUDA;
  }
  if (host_st) *host_st = tmp;
  return tmp.code;
}

namespace {

// Bump allocator over the caller's workspace; with base == nullptr it only
// measures, so the *_workspace_bytes queries and the carving share one layout.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(int64_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += static_cast<size_t>(std::max<int64_t>(count, 1)) * sizeof(T);
    return p;
  }
  size_t bytes() const { return (off + 255) & ~static_cast<size_t>(255); }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_layer(int64_t out, int64_t in, int bits, int g) {
  if (out < 1 || in < 8 || in % 8 != 0) return PIQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4 || g < 1) return PIQ_ERR_INVALID_ARG;
  if (in > (int64_t)1 << 20 || out > (int64_t)1 << 24) return PIQ_ERR_INVALID_ARG;
  return PIQ_OK;
}

// ------------------------------------------------------------- phase timing
constexpr int kMaxPhases = 8;
const char* kPhaseNames[2][kMaxPhases] = {
    {"hessian", "act_order", "factor", "sweep", "pack", "error", nullptr, nullptr},
    {"colstats", "quant_delta", "error_gemm", "select_pack", nullptr, nullptr, nullptr, nullptr}};

struct Timing {
  bool enabled = false;
  int kind = 0;  // 0 gptq, 1 awq
  int n = 0;
  cudaEvent_t ev[kMaxPhases + 1] = {};
  bool created = false;
  double last_ms[kMaxPhases] = {};
  int last_n = 0;
  int last_kind = 0;
  // digit GEMM launches of the current call: event pairs and their work
  bool in_call = false;
  std::vector<cudaEvent_t> gev;  // 2 per slot, created on demand
  std::vector<double> gops;
  int gn = 0;
  double last_gemm_ms = 0.0, last_gemm_ops = 0.0;
  int last_gemm_n = 0;
};
Timing g_timing;
std::mutex g_timing_mu;
constexpr int kMaxGemmSlots = 8192;

}  // namespace

int gemm_timing_begin(cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (!g_timing.enabled || !g_timing.in_call || g_timing.gn >= kMaxGemmSlots) return -1;
  const int slot = g_timing.gn;
  while (static_cast<int>(g_timing.gev.size()) < 2 * (slot + 1)) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    g_timing.gev.push_back(e);
  }
  if (static_cast<int>(g_timing.gops.size()) <= slot) g_timing.gops.resize(slot + 1);
  if (cudaEventRecord(g_timing.gev[2 * slot], stream) != cudaSuccess) return -1;
  ++g_timing.gn;
  return slot;
}

void gemm_timing_end(int slot, cudaStream_t stream, double int8_ops) {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  cudaEventRecord(g_timing.gev[2 * slot + 1], stream);
  g_timing.gops[slot] = int8_ops;
}

namespace {

struct PhaseClock {
  bool on;
  cudaStream_t s;
  int idx = 0;
  PhaseClock(int kind, cudaStream_t stream) : on(false), s(stream) {
    std::lock_guard<std::mutex> lock(g_timing_mu);
    if (!g_timing.enabled) return;
    if (!g_timing.created) {
      for (auto& e : g_timing.ev)
        if (cudaEventCreate(&e) != cudaSuccess) return;
      g_timing.created = true;
    }
    g_timing.kind = kind;
    g_timing.in_call = true;
    g_timing.gn = 0;
    on = true;
    cudaEventRecord(g_timing.ev[0], s);
  }
  void mark() {  // end of the current phase
    if (!on || idx >= kMaxPhases) return;
    cudaEventRecord(g_timing.ev[++idx], s);
  }
  void finish() {  // after the stream synchronized
    if (!on) return;
    std::lock_guard<std::mutex> lock(g_timing_mu);
    for (int i = 0; i < idx; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, g_timing.ev[i], g_timing.ev[i + 1]);
      g_timing.last_ms[i] = ms;
    }
    g_timing.last_n = idx;
    g_timing.last_kind = g_timing.kind;
    double gms = 0.0, gops = 0.0;
    for (int i = 0; i < g_timing.gn; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, g_timing.gev[2 * i], g_timing.gev[2 * i + 1]);
      gms += ms;
      gops += g_timing.gops[i];
    }
    g_timing.last_gemm_ms = gms;
    g_timing.last_gemm_ops = gops;
    g_timing.last_gemm_n = g_timing.gn;
    g_timing.in_call = false;
    g_timing.gn = 0;
  }
};

#define PIQ_TRY(expr)             \
  do {                            \
    const int rc_ = (expr);       \
    if (rc_ != PIQ_OK) return rc_; \
  } while (0)

// ------------------------------------------------------------ layouts
struct FactorWs {
  DeviceStatus* st;
  float* work;
};
FactorWs carve_factor(Carver& c, int64_t in) {
  FactorWs w;
  w.st = c.take<DeviceStatus>(1);
  w.work = c.take<float>(factor_workspace_floats(in));
  return w;
}

struct SweepWs {
  DeviceStatus* st;
  float* Wq;
  float* Err;
};
SweepWs carve_sweep(Carver& c, int64_t out, int64_t in) {
  SweepWs w;
  w.st = c.take<DeviceStatus>(1);
  w.Wq = c.take<float>(out * in);
  w.Err = c.take<float>(out * kSweepB);
  return w;
}

// Everything of a GPTQ call after H (and the act-order key) exist.
struct FromHWs {
  DeviceStatus* st;
  void* fwork;     // FP64 factor (L first); later the error's bf16 split of H
  float* Wq;       // W in quantization order (read by the sweep); later the bf16 split of D
  int8_t* codes;
  float* qscale;
  float* dW;       // W - What (fp32, memory order)
  int32_t* perm;
  int32_t* invperm;
  double* partials;
  double* err;
  Sweep64Ws sw;
};
FromHWs carve_from_h(Carver& c, int64_t out, int64_t in, int g) {
  FromHWs w;
  w.st = c.take<DeviceStatus>(1);
  w.fwork = c.take<uint8_t>(factor64_workspace_bytes(in));
  w.Wq = c.take<float>(out * in);
  w.codes = c.take<int8_t>(out * in);
  w.qscale = c.take<float>(out * ceil_div(in, 1));  // sized for g >= 1
  w.dW = c.take<float>(out * in);
  w.perm = c.take<int32_t>(in);
  w.invperm = c.take<int32_t>(in);
  w.partials = c.take<double>(err_via_h_partials(out, in));
  w.err = c.take<double>(1);
  uint8_t* sb = c.take<uint8_t>(sweep64_workspace_bytes(out, in, g));
  carve_sweep64(sb, out, in, g, &w.sw);
  return w;
}

struct StatsWs {
  double* colpart;
};
StatsWs carve_stats(Carver& c, int64_t n, int64_t in) {
  StatsWs w;
  w.colpart = c.take<double>(static_cast<int64_t>(colstats_splits(n, in)) * in * 2);
  return w;
}

struct GptqWs {
  double* H;       // X^T X (FP64-grade sums), kept for the output error
  double* sumsq;   // act-order key
  StatsWs stats;
  FromHWs fh;
};
GptqWs carve_gptq(Carver& c, int64_t out, int64_t in, int64_t n, int g, int act_order) {
  GptqWs w;
  w.H = c.take<double>(in * in);
  w.sumsq = c.take<double>(in);
  if (act_order)
    w.stats = carve_stats(c, n, in);
  else
    w.stats.colpart = c.take<double>(1);
  w.fh = carve_from_h(c, out, in, g);
  return w;
}

struct AwqWs {
  DeviceStatus* st;
  double* colpart;
  double* mean_abs;
  float* alphas;
  float* s_table;
  uint16_t* dW;
  double* partials;
  double* err;
  int* best;
  float* best_alpha;
  int8_t* codes;
  float* qscale;
};
AwqWs carve_awq(Carver& c, int64_t out, int64_t in, int64_t n, int n_alpha) {
  AwqWs w;
  w.st = c.take<DeviceStatus>(1);
  w.colpart = c.take<double>(static_cast<int64_t>(colstats_splits(n, in)) * in * 2);
  w.mean_abs = c.take<double>(in);
  w.alphas = c.take<float>(64);
  w.s_table = c.take<float>(2 * static_cast<int64_t>(n_alpha) * in);  // s, then 1/s
  w.dW = c.take<uint16_t>(static_cast<int64_t>(n_alpha) * out * in);
  w.partials = c.take<double>(sumsq_partials_count(n, out, n_alpha));
  w.err = c.take<double>(64);
  w.best = c.take<int>(1);
  w.best_alpha = c.take<float>(1);
  w.codes = c.take<int8_t>(out * in);
  w.qscale = c.take<float>(out * in);  // sized for g >= 1
  return w;
}

struct RtnWs {
  int8_t* codes;
  float* qscale;
};
RtnWs carve_rtn(Carver& c, int64_t out, int64_t in) {
  RtnWs w;
  w.codes = c.take<int8_t>(out * in);
  w.qscale = c.take<float>(out * in);  // sized for g >= 1
  return w;
}

// Route of piq_layer_output_error, in BF16 tensor-core flops: through X,
// 2 n in out; through H, n in^2 for X^T X plus three bf16 passes over the
// triangular out x in x in product, 3 out in^2.
bool error_route_h(int64_t out, int64_t in, int64_t n) {
  const double via_x = 2.0 * n * in * out;
  const double via_h = static_cast<double>(n) * in * in + 3.0 * out * in * in;
  return via_h < via_x;
}

struct ErrWs {
  DeviceStatus* st;
  uint16_t* dW;      // X route: bf16 delta
  float* dW32;       // H route: fp32 delta, H and the bf16 splits
  float* H;
  uint16_t* dsplit;
  uint16_t* hsplit;
  double* partials;
  double* err;
};
ErrWs carve_err(Carver& c, int64_t out, int64_t in, int64_t n) {
  ErrWs w{};
  w.st = c.take<DeviceStatus>(1);
  if (error_route_h(out, in, n)) {
    w.dW32 = c.take<float>(out * in);
    w.H = c.take<float>(in * in);
    w.dsplit = c.take<uint16_t>(2 * out * in);
    w.hsplit = c.take<uint16_t>(2 * in * in);
    w.partials = c.take<double>(err_via_h_partials(out, in));
  } else {
    w.dW = c.take<uint16_t>(out * in);
    w.partials = c.take<double>(sumsq_partials_count(n, out, 1));
  }
  w.err = c.take<double>(1);
  return w;
}

int check_ws(void* ws, size_t have, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PIQ_ERR_INVALID_ARG;
  return have >= need ? PIQ_OK : PIQ_ERR_WORKSPACE_TOO_SMALL;
}

size_t gptq_ws_bytes(int64_t out, int64_t in, int64_t n, int g, int act_order) {
  Carver c(nullptr);
  carve_gptq(c, out, in, n, g, act_order ? 1 : 0);
  return c.bytes();
}

// GPTQ of one layer; with s_ch, of the scaled layer (W diag(s), X diag(1/s)):
// H' = diag(1/s) X^T X diag(1/s), the act-order key diag(H'), the sweep over
// W diag(s), and the error of What = code * scale / s through H' with
// D' = W diag(s) - code * fp16(scale), since X' D'^T = X (W - What)^T.
// With zeros, every group gets a scale and a zero-point (asymmetric groups):
// the sweep writes the zero-points there and the pack stores code + zero.
// Steps 2-6 of GPTQ from a given H (upper triangle, fp64) and, for act-order,
// its key sumsq (diag(H) in exact FP64 sums).  H is read only, except that
// with s_ch it was scaled in place by the caller.
int gptq_core(const float* W, int64_t out, int64_t in, const double* H, const double* sumsq,
              const float* s_ch, int bits, int g, float damp, int act_order, uint32_t* qweight,
              uint16_t* scales, uint8_t* zeros, int32_t* perm, int32_t* g_idx, double* out_err,
              const FromHWs& w, PhaseClock& clk, cudaStream_t s) {
  // 2. quantization order
  const int32_t* qperm = nullptr;
  const int32_t* qinv = nullptr;
  if (act_order) {
    PIQ_TRY(launch_act_order_perm(sumsq, in, w.perm, w.invperm, s));
    qperm = w.perm;
    qinv = w.invperm;
  }
  if (perm) {
    if (act_order)
      PIQ_TRY(cuda_rc(cudaMemcpyAsync(perm, w.perm, sizeof(int32_t) * in, cudaMemcpyDeviceToDevice, s)));
    else
      PIQ_TRY(launch_identity_perm(in, perm, nullptr, s));
  }
  clk.mark();
  // 3. damping + the FP64 factor L of J H_d J (H is kept for the error)
  double* L = nullptr;
  PIQ_TRY(run_factor64(H, in, damp, qperm, w.fwork, &L, w.st, s));
  clk.mark();
  // 4. the sweep on R = J L J over the permuted (and scaled) copy of W
  PIQ_TRY(launch_gather_columns(W, out, in, qperm, s_ch, w.Wq, s));
  PIQ_TRY(run_gptq_sweep64(w.Wq, out, in, L, bits, g, w.codes, w.qscale, zeros, w.sw, w.st, s));
  clk.mark();
  // 5. pack (+ D = W diag(s) - What' for the error)
  PIQ_TRY(launch_pack(w.codes, w.qscale, zeros, qinv, out, in, bits, g, W, s_ch, qweight, scales,
                      nullptr, out_err ? w.dW : nullptr, g_idx, s));
  clk.mark();
  // 6. output error ||X D^T||^2 = 2 sum_r D_r Hu D_r^T, from H
  //    (scratch: the sweep copy, and the factor's region)
  if (out_err)
    PIQ_TRY(run_error_via_h(w.dW, out, in, H, reinterpret_cast<uint16_t*>(w.Wq),
                            reinterpret_cast<uint16_t*>(w.fwork), w.partials, w.err, w.st, s));
  clk.mark();
  double e = 0.0;
  if (out_err)
    PIQ_TRY(cuda_rc(cudaMemcpyAsync(&e, w.err, sizeof(double), cudaMemcpyDeviceToHost, s)));
  const int rc = finish_call(w.st, s, nullptr);
  clk.finish();
  if (out_err) *out_err = e;
  return rc;
}

int gptq_layer(const float* W, int64_t out, int64_t in, const uint16_t* X, int64_t n,
               const float* s_ch, int bits, int g, float damp, int act_order, uint32_t* qweight,
               uint16_t* scales, uint8_t* zeros, int32_t* perm, int32_t* g_idx, double* out_err,
               void* workspace, size_t ws_bytes, cudaStream_t s) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (W == nullptr || X == nullptr || qweight == nullptr || scales == nullptr || n < 1 ||
      !(damp >= 0.f) || !aligned16(W) || !aligned16(X) || !aligned16(qweight))
    return PIQ_ERR_INVALID_ARG;
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  PIQ_TRY(check_ws(workspace, ws_bytes, gptq_ws_bytes(out, in, n, g, act_order)));
  Carver c(workspace);
  GptqWs w = carve_gptq(c, out, in, n, g, act_order ? 1 : 0);
  PhaseClock clk(0, s);

  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.fh.st, 0, sizeof(DeviceStatus), s)));
  // 1. H = X^T X on the tensor cores (scaled to H' for the AWQ-scaled layer), and
  //    the act-order key: exact FP64 column sums of squares (scaled alike)
  PIQ_TRY(launch_syrk64(X, n, in, w.H, w.fh.st, s));
  if (s_ch) PIQ_TRY(launch_scale_upper(w.H, in, s_ch, w.fh.st, s));
  if (act_order) {
    PIQ_TRY(launch_colstats(X, n, in, w.stats.colpart, colstats_splits(n, in), nullptr, w.sumsq,
                            s));
    if (s_ch) PIQ_TRY(launch_scale_sumsq(w.sumsq, in, s_ch, s));
  }
  clk.mark();
  return gptq_core(W, out, in, w.H, w.sumsq, s_ch, bits, g, damp, act_order, qweight, scales,
                   zeros, perm, g_idx, out_err, w.fh, clk, s);
}

}  // namespace
}  // namespace piq

using namespace piq;

extern "C" {

const char* piq_status_string(int status) {
  switch (status) {
    case PIQ_OK: return "ok";
    case PIQ_ERR_INVALID_ARG: return "invalid argument";
    case PIQ_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case PIQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case PIQ_ERR_CUDA: return "CUDA error";
    case PIQ_ERR_TIMEOUT: return "bounded device wait timed out";
    case PIQ_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    default: return "unknown status";
  }
}

int piq_hessian_bytes(int64_t in, size_t* bytes) {
  if (bytes == nullptr || in < 1) return PIQ_ERR_INVALID_ARG;
  *bytes = static_cast<size_t>(in) * static_cast<size_t>(in) * sizeof(float);
  return PIQ_OK;
}

int piq_hessian(const uint16_t* X, int64_t n, int64_t in, float* H, int accumulate,
                void* stream) {
  if (X == nullptr || H == nullptr || !aligned16(X) || !aligned16(H)) return PIQ_ERR_INVALID_ARG;
  if (n < 1 || in < 8 || in % 8 != 0) return PIQ_ERR_INVALID_ARG;
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  return launch_syrk_xtx(X, n, in, H, accumulate, nullptr, static_cast<cudaStream_t>(stream));
}

int piq_upper_factor_workspace_bytes(int64_t in, size_t* bytes) {
  if (bytes == nullptr || in < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_factor(c, in);
  *bytes = c.bytes();
  return PIQ_OK;
}

int piq_upper_factor(const float* H, int64_t in, float damp, const int32_t* perm, float* U,
                     double* lambda_out, void* workspace, size_t ws_bytes, void* stream) {
  if (H == nullptr || U == nullptr || in < 1 || !(damp >= 0.f)) return PIQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_upper_factor_workspace_bytes(in, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  Carver c(workspace);
  FactorWs w = carve_factor(c, in);
  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.st, 0, sizeof(DeviceStatus), s)));
  PIQ_TRY(run_upper_factor(H, in, damp, perm, U, w.work, w.st, s));
  DeviceStatus hs;
  const int rc = finish_call(w.st, s, &hs);
  if (lambda_out) *lambda_out = hs.lambda;
  return rc;
}

int piq_gptq_sweep_workspace_bytes(int64_t out, int64_t in, size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_sweep(c, out, in);
  *bytes = c.bytes();
  return PIQ_OK;
}

int piq_gptq_sweep(const float* Wp, int64_t out, int64_t in, const float* U, int bits, int g,
                   int8_t* codes, float* qscale, void* workspace, size_t ws_bytes,
                   void* stream) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (Wp == nullptr || U == nullptr || codes == nullptr || qscale == nullptr)
    return PIQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_gptq_sweep_workspace_bytes(out, in, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  Carver c(workspace);
  SweepWs w = carve_sweep(c, out, in);
  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.st, 0, sizeof(DeviceStatus), s)));
  PIQ_TRY(cuda_rc(cudaMemcpyAsync(w.Wq, Wp, sizeof(float) * out * in, cudaMemcpyDeviceToDevice, s)));
  PIQ_TRY(run_gptq_sweep(w.Wq, out, in, U, bits, g, codes, qscale, nullptr, w.Err, w.st, s));
  return finish_call(w.st, s, nullptr);
}

int piq_gptq_workspace_bytes(int64_t out, int64_t in, int64_t n, int g, int act_order,
                             size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1 || n < 1 || g < 1) return PIQ_ERR_INVALID_ARG;
  *bytes = gptq_ws_bytes(out, in, n, g, act_order);
  return PIQ_OK;
}

int gptq_quantize_layer(const float* W, int64_t out, int64_t in, const uint16_t* X, int64_t n,
                        int bits, int g, float damp, int act_order, uint32_t* qweight,
                        uint16_t* scales, int32_t* perm, int32_t* g_idx, double* out_err,
                        void* workspace, size_t ws_bytes, void* stream) {
  return gptq_layer(W, out, in, X, n, nullptr, bits, g, damp, act_order, qweight, scales, nullptr,
                    perm, g_idx, out_err, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int gptq_quantize_layer_asym(const float* W, int64_t out, int64_t in, const uint16_t* X,
                             int64_t n, int bits, int g, float damp, int act_order,
                             uint32_t* qweight, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                             int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (zeros == nullptr) return PIQ_ERR_INVALID_ARG;
  return gptq_layer(W, out, in, X, n, nullptr, bits, g, damp, act_order, qweight, scales, zeros,
                    perm, g_idx, out_err, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int piq_layer_statistics_workspace_bytes(int64_t n, int64_t in, size_t* bytes) {
  if (bytes == nullptr || n < 1 || in < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  c.take<DeviceStatus>(1);
  carve_stats(c, n, in);
  *bytes = c.bytes();
  return PIQ_OK;
}

int piq_layer_statistics(const uint16_t* X, int64_t n, int64_t in, double* H, double* sumsq,
                         void* workspace, size_t ws_bytes, void* stream) {
  if (X == nullptr || H == nullptr || n < 1 || in < 8 || in % 8 != 0 || !aligned16(X) ||
      !aligned16(H) || in > (int64_t)1 << 20)
    return PIQ_ERR_INVALID_ARG;
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_layer_statistics_workspace_bytes(n, in, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  DeviceStatus* st = c.take<DeviceStatus>(1);
  StatsWs w = carve_stats(c, n, in);
  PIQ_TRY(cuda_rc(cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s)));
  PIQ_TRY(launch_syrk64(X, n, in, H, st, s));
  if (sumsq) PIQ_TRY(launch_colstats(X, n, in, w.colpart, colstats_splits(n, in), nullptr, sumsq, s));
  return finish_call(st, s, nullptr);
}

int piq_gptq_from_h_workspace_bytes(int64_t out, int64_t in, int g, size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1 || g < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_from_h(c, out, in, g);
  *bytes = c.bytes();
  return PIQ_OK;
}

int gptq_quantize_rows_from_h(const float* W, int64_t out, int64_t in, const double* H,
                              const double* sumsq, int bits, int g, float damp, int act_order,
                              uint32_t* qweight, uint16_t* scales, uint8_t* zeros, int32_t* perm,
                              int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                              void* stream) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (W == nullptr || H == nullptr || qweight == nullptr || scales == nullptr ||
      !(damp >= 0.f) || !aligned16(W) || !aligned16(H) || !aligned16(qweight) ||
      (act_order && sumsq == nullptr))
    return PIQ_ERR_INVALID_ARG;
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_gptq_from_h_workspace_bytes(out, in, g, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver c(workspace);
  FromHWs w = carve_from_h(c, out, in, g);
  PhaseClock clk(0, s);
  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.st, 0, sizeof(DeviceStatus), s)));
  clk.mark();  // no H phase: H is given
  return gptq_core(W, out, in, H, sumsq, nullptr, bits, g, damp, act_order, qweight, scales,
                   zeros, perm, g_idx, out_err, w, clk, s);
}

int awq_gptq_quantize_layer(const float* W, int64_t out, int64_t in, const uint16_t* X,
                            int64_t n, const float* s_ch, int bits, int g, float damp,
                            int act_order, uint32_t* qweight, uint16_t* scales, int32_t* perm,
                            int32_t* g_idx, double* out_err, void* workspace, size_t ws_bytes,
                            void* stream) {
  if (s_ch == nullptr || !aligned16(s_ch)) return PIQ_ERR_INVALID_ARG;
  return gptq_layer(W, out, in, X, n, s_ch, bits, g, damp, act_order, qweight, scales, nullptr,
                    perm, g_idx, out_err, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int piq_awq_workspace_bytes(int64_t out, int64_t in, int64_t n, int n_alpha, size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1 || n < 1 || n_alpha < 1 || n_alpha > 64)
    return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_awq(c, out, in, n, n_alpha);
  *bytes = c.bytes();
  return PIQ_OK;
}

int awq_search_layer(const float* W, int64_t out, int64_t in, const uint16_t* X, int64_t n,
                     int bits, int g, const float* alpha_grid, int n_alpha, float* best_alpha,
                     float* s_out, uint32_t* qweight, uint16_t* scales, double* err_per_alpha,
                     void* workspace, size_t ws_bytes, void* stream) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (W == nullptr || X == nullptr || alpha_grid == nullptr || s_out == nullptr ||
      qweight == nullptr || scales == nullptr || n < 1 || n_alpha < 1 || n_alpha > 64 ||
      !aligned16(W) || !aligned16(X) || !aligned16(qweight))
    return PIQ_ERR_INVALID_ARG;
  for (int a = 0; a < n_alpha; ++a)
    if (!(alpha_grid[a] == alpha_grid[a])) return PIQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_awq_workspace_bytes(out, in, n, n_alpha, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  Carver c(workspace);
  AwqWs w = carve_awq(c, out, in, n, n_alpha);
  PhaseClock clk(1, s);

  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.st, 0, sizeof(DeviceStatus), s)));
  PIQ_TRY(cuda_rc(cudaMemcpyAsync(w.alphas, alpha_grid, sizeof(float) * n_alpha,
                                  cudaMemcpyHostToDevice, s)));
  // 1. mean |x_j|
  PIQ_TRY(launch_colstats(X, n, in, w.colpart, colstats_splits(n, in), w.mean_abs, nullptr, s));
  clk.mark();
  // 2. s = m^alpha for the grid, and D_alpha = W - code * scale / s
  PIQ_TRY(launch_awq_scale_table(w.mean_abs, in, w.alphas, n_alpha, w.s_table, s));
  PIQ_TRY(launch_awq_delta(W, out, in, bits, g, w.s_table, n_alpha, w.dW, s));
  clk.mark();
  // 3. E_alpha = ||X D_alpha^T||^2, every alpha in one tensor-core launch
  PIQ_TRY(launch_err_sumsq(X, n, in, w.dW, out, n_alpha, w.partials, w.st, s));
  PIQ_TRY(launch_reduce_partials(w.partials, n, out, n_alpha, w.err, s));
  clk.mark();
  // 4. first minimum, re-quantize at it, pack
  PIQ_TRY(launch_argmin(w.err, n_alpha, w.alphas, w.best, w.best_alpha, s));
  PIQ_TRY(launch_group_quant(W, out, in, bits, g, w.s_table, w.best, w.codes, w.qscale, s_out, s));
  PIQ_TRY(launch_pack(w.codes, w.qscale, nullptr, nullptr, out, in, bits, g, nullptr, nullptr, qweight,
                      scales, nullptr, nullptr, nullptr, s));
  clk.mark();
  double errs[64];
  float ba = 0.f;
  PIQ_TRY(cuda_rc(cudaMemcpyAsync(errs, w.err, sizeof(double) * n_alpha, cudaMemcpyDeviceToHost, s)));
  PIQ_TRY(cuda_rc(cudaMemcpyAsync(&ba, w.best_alpha, sizeof(float), cudaMemcpyDeviceToHost, s)));
  const int rc = finish_call(w.st, s, nullptr);
  clk.finish();
  if (err_per_alpha) std::memcpy(err_per_alpha, errs, sizeof(double) * n_alpha);
  if (best_alpha) *best_alpha = ba;
  return rc;
}

int piq_rtn_workspace_bytes(int64_t out, int64_t in, size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_rtn(c, out, in);
  *bytes = c.bytes();
  return PIQ_OK;
}

int piq_rtn_quantize_layer(const float* W, int64_t out, int64_t in, int bits, int g,
                           uint32_t* qweight, uint16_t* scales, void* workspace,
                           size_t ws_bytes, void* stream) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (W == nullptr || qweight == nullptr || scales == nullptr || !aligned16(W) ||
      !aligned16(qweight))
    return PIQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_rtn_workspace_bytes(out, in, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  Carver c(workspace);
  RtnWs w = carve_rtn(c, out, in);
  PIQ_TRY(launch_group_quant(W, out, in, bits, g, nullptr, nullptr, w.codes, w.qscale, nullptr, s));
  return launch_pack(w.codes, w.qscale, nullptr, nullptr, out, in, bits, g, nullptr, nullptr, qweight,
                     scales, nullptr, nullptr, nullptr, s);
}

int piq_output_error_workspace_bytes(int64_t out, int64_t in, int64_t n, size_t* bytes) {
  if (bytes == nullptr || out < 1 || in < 1 || n < 1) return PIQ_ERR_INVALID_ARG;
  Carver c(nullptr);
  carve_err(c, out, in, n);
  *bytes = c.bytes();
  return PIQ_OK;
}

int piq_layer_output_error(const float* W, int64_t out, int64_t in, const uint32_t* qweight,
                           const uint16_t* scales, const uint8_t* zeros, const int32_t* g_idx,
                           const float* s_ch, int bits, int g, const uint16_t* X, int64_t n,
                           double* out_err, void* workspace, size_t ws_bytes, void* stream) {
  PIQ_TRY(check_layer(out, in, bits, g));
  if (W == nullptr || qweight == nullptr || scales == nullptr || X == nullptr ||
      out_err == nullptr || n < 1 || !aligned16(W) || !aligned16(X) || !aligned16(qweight))
    return PIQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PIQ_TRY(injected_fault());
  DeviceInfo info;
  PIQ_TRY(device_info(&info));
  size_t need = 0;
  piq_output_error_workspace_bytes(out, in, n, &need);
  PIQ_TRY(check_ws(workspace, ws_bytes, need));
  Carver c(workspace);
  ErrWs w = carve_err(c, out, in, n);
  PIQ_TRY(cuda_rc(cudaMemsetAsync(w.st, 0, sizeof(DeviceStatus), s)));
  if (error_route_h(out, in, n)) {
    PIQ_TRY(launch_dequant_delta(W, out, in, qweight, scales, zeros, g_idx, s_ch, bits, g,
                                 nullptr, w.dW32, w.st, s));
    PIQ_TRY(launch_syrk_xtx(X, n, in, w.H, 0, w.st, s));
    PIQ_TRY(run_error_via_h(w.dW32, out, in, w.H, w.dsplit, w.hsplit, w.partials, w.err, w.st,
                            s));
  } else {
    PIQ_TRY(launch_dequant_delta(W, out, in, qweight, scales, zeros, g_idx, s_ch, bits, g, w.dW,
                                 nullptr, w.st, s));
    PIQ_TRY(launch_err_sumsq(X, n, in, w.dW, out, 1, w.partials, w.st, s));
    PIQ_TRY(launch_reduce_partials(w.partials, n, out, 1, w.err, s));
  }
  double e = 0.0;
  PIQ_TRY(cuda_rc(cudaMemcpyAsync(&e, w.err, sizeof(double), cudaMemcpyDeviceToHost, s)));
  const int rc = finish_call(w.st, s, nullptr);
  *out_err = e;
  return rc;
}

int piq_set_timing(int enable) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  g_timing.enabled = enable != 0;
  return PIQ_OK;
}

int piq_last_phase_times(double* ms, int max_phases, int* n_phases) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  const int n = std::min(max_phases, g_timing.last_n);
  for (int i = 0; i < n; ++i) ms[i] = g_timing.last_ms[i];
  if (n_phases) *n_phases = g_timing.last_n;
  return PIQ_OK;
}

int piq_last_gemm_stats(double* ms, double* int8_ops, int* launches) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (ms) *ms = g_timing.last_gemm_ms;
  if (int8_ops) *int8_ops = g_timing.last_gemm_ops;
  if (launches) *launches = g_timing.last_gemm_n;
  return PIQ_OK;
}

uint64_t piq_kernel_launches(void) { return g_launches.load(); }

uint64_t piq_simt_gemm_fallbacks(void) { return simt_gemm_fallbacks(); }

const char* piq_last_cuda_error(void) {
  std::lock_guard<std::mutex> lock(g_err_mu);
  return g_err_text;
}

const char* piq_phase_name(int i) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (i < 0 || i >= kMaxPhases) return nullptr;
  return kPhaseNames[g_timing.last_kind][i];
}

}  // extern "C"
