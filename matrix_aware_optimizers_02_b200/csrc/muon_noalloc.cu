// mao_muon_step_noalloc: the Muon step for callers that cannot allocate device
// memory for its scratch workspace.
//
// The scratch is one file-scope __device__ array of MAO_NOALLOC_SCRATCH_BYTES
// that every device loading the library holds until the process exits.  Host
// code cannot use the array's name as a device address (on the host it names a
// stand-in object), so the device address is fetched once per device with
// cudaGetSymbolAddress, with that device current, on the first call made there,
// and cached.  The step itself is the unchanged mao_muon_step given that
// address as its workspace.
#include <mutex>

#include "host_common.h"

namespace {

constexpr size_t kScratchBytes = MAO_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

}  // namespace

// Device address of the scratch array on the current device, looked up on the
// first use there.
static mao_status scratch_address(void** out) {
  int dev = 0;
  MAO_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MAO_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess || a == nullptr) return MAO_ERR_CUDA;
    g_scratch_addr[dev] = a;
  }
  *out = g_scratch_addr[dev];
  return MAO_OK;
}

extern "C" mao_status mao_muon_step_noalloc(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p,
                                           mao_stats* stats, mao_stream_t stream) {
  size_t need = 0;
  MAO_TRY(mao_muon_workspace_size(mats, count, p, &need));
  if (need > kScratchBytes) return MAO_ERR_WORKSPACE;
  void* addr = nullptr;
  MAO_TRY(scratch_address(&addr));
  // The status word at the start of the scratch is cleared by the step itself;
  // nothing else in the scratch needs to start at zero.
  return mao_muon_step(mats, count, p, addr, kScratchBytes, stats, stream);
}

// The status word of the last mao_muon_step_noalloc on the current device lives at
// the start of the scratch array, whose address only this file knows.
extern "C" mao_status mao_muon_noalloc_status(mao_stream_t stream, int32_t* where) {
  void* addr = nullptr;
  MAO_TRY(scratch_address(&addr));
  return mao_workspace_status(addr, stream, where);
}
