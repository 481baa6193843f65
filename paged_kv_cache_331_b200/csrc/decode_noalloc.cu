// pa_decode_noalloc: paged decode whose split-KV scratch lives in a fixed
// array inside this library instead of a buffer the caller provides.
//
// Who needs it: callers that cannot hand the library a device allocation of
// their own -- for example a plugin running inside a host process that owns
// and pre-partitions all device memory, or a C caller with no access to the
// allocator that manages its device memory.  They still pass every input and
// output; only the partial results of the split-KV pass go to the array below.
//
// Costs and rules:
//  * Every GPU that loads this library reserves kScratchBytes of device
//    memory for the array, for as long as the library stays loaded.
//  * All calls on a device share the one array.  Calls whose kernels can
//    overlap on that device (different streams, or different host threads
//    without ordering) race on it and produce garbage; order such calls.
//  * The array keeps whatever the last call left in it.  Nothing here needs
//    it to start at zero: every partial the merge pass reads is written
//    earlier in the same call.
//  * The device address of the array is looked up on the first call made on
//    each device (with that device current); that first call should happen
//    before any stream capture begins on the device.  The address is kept
//    until the library is unloaded, so it is stale after the device's
//    primary context is reset (cudaDeviceReset); a lookup that failed is
//    tried again on the next call.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace pa {
namespace {

constexpr size_t kScratchBytes = PA_DECODE_NOALLOC_SCRATCH_BYTES;

// In host code this name is only a stand-in for the device array; kernels get
// the address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  A successful
// lookup is kept for the library's lifetime (it stays valid until the
// device's primary context is reset); a failed one is not kept, so the next
// call tries again.  Returns nullptr and records a message on failure.
void* scratch_for_current_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_last_error("decode_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    set_last_error("decode_noalloc: device ordinal %d is beyond the %d this build tracks", dev, kMaxDevices);
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) {
      set_last_error("decode_noalloc: cudaGetSymbolAddress failed on device %d: %s", dev, cudaGetErrorString(e));
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs,
                                       int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                       int32_t num_blocks, float scale, int32_t kv_chunk_size, void* stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                               block_size, kv_chunk_size);
  if (need > pa::kScratchBytes) {
    pa::set_last_error(
        "decode_noalloc: this shape needs %zu bytes of split-KV scratch but the library's static array holds %zu; "
        "use pa_decode with a caller-provided workspace, or a larger kv_chunk_size",
        need, pa::kScratchBytes);
    return PA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0 && !(scratch = pa::scratch_for_current_device())) return PA_ERR_CUDA;
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                   num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, kv_chunk_size, scratch,
                   need > 0 ? pa::kScratchBytes : 0, stream);
}
