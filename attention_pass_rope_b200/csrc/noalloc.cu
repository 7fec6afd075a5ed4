// Forward entry point for callers that cannot allocate device memory.
//
// ttt_attn_fwd needs a caller-provided workspace.  Some callers have no way to get
// one: a plugin inside a host framework that owns every device allocation and gives
// its extensions none, or a latency-critical loop where calling cudaMalloc (which
// can synchronise the whole device) is not acceptable.  ttt_attn_fwd_noalloc runs
// the same forward with its scratch in a fixed array that lives in the library's
// own device memory instead; it calls no cudaMalloc, cudaFree or allocating library
// routine.
//
// The array is a file-scope __device__ variable, so every GPU that loads the library
// holds its kNoallocScratchBytes until the process exits.  In host code the
// variable's name is only a host-side handle, never a device address: the device
// address is obtained with cudaGetSymbolAddress, once per device, with that device
// current, on the first call made on it (that first call should therefore come
// before any stream capture), and cached.
//
// All calls on a device share the one array and it keeps whatever the last call left
// in it.  The forward clears what must start at zero (its status word) itself.  Two
// calls whose work overlaps on the GPU (different streams, no ordering between
// them) race on the array and give undefined results; order them on one stream.
//
// The forward's bounded in-kernel waits record a timeout in the first word of the
// array, as the workspace forward does in the first word of its workspace; this
// caller has no pointer to it, so ttt_attn_fwd_noalloc_status reads it instead.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ttt_attn.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
ttt_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return TTT_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TTT_OK;
}

}  // namespace

extern "C" ttt_status ttt_attn_fwd_noalloc_status(void* stream, uint32_t* detail) {
  void* scratch = nullptr;
  const ttt_status st = scratch_on_current_device(&scratch);
  if (st != TTT_OK) return st;
  return ttt_attn_device_status(scratch, stream, detail);
}

extern "C" ttt_status ttt_attn_noalloc_watchdog_selftest(uint64_t budget_ns, void* stream) {
  void* scratch = nullptr;
  const ttt_status st = scratch_on_current_device(&scratch);
  if (st != TTT_OK) return st;
  return ttt_attn_watchdog_selftest(scratch, kNoallocScratchBytes, budget_ns, stream);
}

extern "C" ttt_status ttt_attn_fwd_noalloc(const ttt_attn_desc* desc, const void* q, const void* k, const void* v,
                                           void* o, float* lse, void* stream) {
  const size_t need = ttt_attn_workspace_size(desc, 0);
  if (need == 0) {
    // invalid descriptor: let the regular entry point report which check failed
    return ttt_attn_fwd(desc, q, k, v, o, lse, nullptr, 0, stream);
  }
  if (need > kNoallocScratchBytes) return TTT_ERR_WORKSPACE;
  void* scratch = nullptr;
  const ttt_status st = scratch_on_current_device(&scratch);
  if (st != TTT_OK) return st;
  // the forward's own size: a larger workspace would also get the backward's accumulator zeroed
  return ttt_attn_fwd(desc, q, k, v, o, lse, scratch, need, stream);
}
