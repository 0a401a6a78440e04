// piq_upper_factor_noalloc: the damping + upper-factor step with its scratch in
// a fixed region of device memory that the library owns, for callers that must
// not allocate device memory themselves (see include/piq.h).
//
// The region is a file-scope __device__ array, so every GPU that loads the
// library holds it until the process exits.  Host code never uses the array's
// name as an address: its device address is fetched once per device with
// cudaGetSymbolAddress while that device is current.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace piq {
namespace {

constexpr int64_t kNoAllocMaxIn = PIQ_NOALLOC_MAX_IN;
// status word (256 bytes) + P and X (in x in each) + pair scratch (at most
// (in/2)^2 for in <= 512) + lambda, for the largest supported in
constexpr size_t kNoAllocBytes =
    256 + static_cast<size_t>(2 * kNoAllocMaxIn * kNoAllocMaxIn + 256 * 256 + 64) * 4;

static __device__ __align__(256) unsigned char g_factor_scratch[kNoAllocBytes];

struct ScratchAddr {
  void* ptr = nullptr;
  bool ready = false;
};
ScratchAddr g_addr[64];
std::mutex g_addr_mu;

// Device address of the region for the current device (set up on first use).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PIQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev].ready) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_factor_scratch);
    if (e != cudaSuccess) {
      note_cuda_error(e, "cudaGetSymbolAddress of the fixed factor region");
      return PIQ_ERR_CUDA;
    }
    if (p == nullptr) return PIQ_ERR_CUDA;
    g_addr[dev].ptr = p;
    g_addr[dev].ready = true;
  }
  *out = g_addr[dev].ptr;
  return PIQ_OK;
}

}  // namespace
}  // namespace piq

using namespace piq;

extern "C" int piq_upper_factor_noalloc(const float* H, int64_t in, float damp,
                                        const int32_t* perm, float* U, double* lambda_out,
                                        void* stream) {
  if (H == nullptr || U == nullptr || in < 1 || !(damp >= 0.f)) return PIQ_ERR_INVALID_ARG;
  if (in > kNoAllocMaxIn) return PIQ_ERR_INVALID_ARG;  // larger than the fixed region
  if (256 + static_cast<size_t>(factor_workspace_floats(in)) * 4 > kNoAllocBytes)
    return PIQ_ERR_INVALID_ARG;
  int rc = injected_fault();
  if (rc != PIQ_OK) return rc;
  DeviceInfo info;
  rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  void* base = nullptr;
  rc = scratch_for_current_device(&base);
  if (rc != PIQ_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus* st = static_cast<DeviceStatus*>(base);
  float* work = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + 256);
  // the region keeps the previous call's contents: only the status word must
  // start at zero (every other byte is written before it is read)
  rc = cuda_rc(cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s));
  if (rc != PIQ_OK) return rc;
  rc = run_upper_factor(H, in, damp, perm, U, work, st, s);
  if (rc != PIQ_OK) return rc;
  DeviceStatus hs;
  rc = finish_call(st, s, &hs);
  if (rc == PIQ_OK && lambda_out) *lambda_out = hs.lambda;
  return rc;
}
