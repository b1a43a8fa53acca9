// mla_decode_noalloc: mla_decode for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside someone else's memory budget and may not call
// cudaMalloc or any allocator on the decode path -- for example a serving engine that
// reserves nearly all HBM for its KV cache up front and forbids allocation during a
// decode step, or a plugin invoked on a stream and memory pool it does not own. Such a
// caller can still pass its inputs and outputs, but not the split workspace.
//
// How: the workspace lives in one file-scope device array of kNoAllocScratchBytes. Every
// GPU that loads this part of the library holds that array until the process exits.
// Host code cannot use the array's name as a device address (it is a host-side stand-in),
// so the first call on each device, with that device current, looks the address up with
// cudaGetSymbolAddress and keeps it. Make that first call before any stream capture.
// All calls on a device share the array and its contents persist between calls. Nothing needs
// clearing: the combine step recomputes each sequence's split from seq_lens and reads only the
// partial slots that the decode kernel of the same call writes (with NaN when a wait ran out),
// so a previous call's leftovers are never read. Calls whose work overlaps on the GPU
// (different streams, or host threads racing) race on the array: serialise them.
#include <atomic>
#include <mutex>

#include "../../include/mla_decode.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)MLA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_mla_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's scratch array, looked up on first use per device (with that
// device current). A failed lookup is not remembered: the next call tries again.
void* scratch_for(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (!p && cudaGetSymbolAddress(&p, g_mla_scratch) == cudaSuccess) g_scratch_ptr[dev].store(p, std::memory_order_release);
  return g_scratch_ptr[dev].load(std::memory_order_relaxed);
}

}  // namespace

extern "C" {

mla_status_t mla_decode_noalloc(const mla_decode_params_t* params, const void* q_lat, const void* q_rope,
                                const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                                const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                                void* stream) {
  size_t need = 0;
  mla_status_t st = mla_decode_workspace_size(params, &need);
  if (st != MLA_OK) return st;
  if (need > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  void* scratch = scratch_for(dev);
  if (!scratch) return MLA_ERR_CUDA;
  return mla_decode(params, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse,
                    scratch, kNoAllocScratchBytes, stream);
}

size_t mla_decode_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

}  // extern "C"
