// piq_wait_selftest: runs out one bounded device wait on purpose.
//
// Every kernel of the library that waits (on a TMA copy, a tensor-core
// commit, another warp role) does so through mbar_wait, which gives up after a
// time limit, records PIQ_ERR_TIMEOUT in the call's status word and lets the
// kernel return normally.  This entry point launches one CTA whose thread 0
// waits, through that same function, on an mbarrier that nothing ever arrives
// on, so the limit is always reached; the host then reads the status word the
// way every other call does.  Nothing faults and the context stays usable.
#include "internal.h"

namespace piq {
namespace {

constexpr int kSelftestWhere = 901;

__global__ void wait_selftest_kernel(DeviceStatus* st) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none comes
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, st, kSelftestWhere);
  __syncthreads();
}

__global__ void init_status_kernel(DeviceStatus* st, uint64_t wait_ns) {
  st->code = PIQ_OK;
  st->where = 0;
  st->lambda = 0.0;
  for (int i = 0; i < 6; ++i) st->aux[i] = 0.0;
  st->wait_ns = wait_ns;
}

}  // namespace
}  // namespace piq

using namespace piq;

extern "C" int piq_wait_selftest(uint64_t wait_ns, int* where_out, void* workspace,
                                 size_t ws_bytes, void* stream) {
  if (wait_ns < 1000 || wait_ns > 10000000000ull) return PIQ_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return PIQ_ERR_INVALID_ARG;
  if (ws_bytes < 256) return PIQ_ERR_WORKSPACE_TOO_SMALL;
  DeviceInfo info;
  int rc = device_info(&info);
  if (rc != PIQ_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus* st = static_cast<DeviceStatus*>(workspace);
  note_launch();
  init_status_kernel<<<1, 1, 0, s>>>(st, wait_ns);
  note_launch();
  wait_selftest_kernel<<<1, 32, 0, s>>>(st);
  if (!launch_ok("wait self-test launch")) return PIQ_ERR_CUDA;
  DeviceStatus hs;
  rc = finish_call(st, s, &hs);
  if (where_out) *where_out = hs.where;
  return rc;
}
