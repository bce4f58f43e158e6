// decode_no_alloc.cu -- pa_decode for callers that cannot allocate device memory.
//
// Some callers can't call cudaMalloc or any allocating routine: for example a
// plug-in running inside a host inference engine that owns every device
// allocation and hands the plug-in no workspace, or a serving runtime that
// forbids device allocation once it has started.  pa_decode_no_alloc gives
// them decode attention without a caller-provided workspace: its scratch is
// the file-scope device array below, which every GPU that loads this library
// holds (PA_DECODE_NO_ALLOC_MAX_BYTES) until the process exits.
//
// Set-up: the first call on a device looks up the array's device address with
// cudaGetSymbolAddress while that device is current, and caches it per device.
// That first call should come before any stream capture.  The cached address
// belongs to the context it was looked up in: after a cudaDeviceReset of the
// device the entry point must not be called again in that process.  In host code the
// array's name is only a host-side stand-in, never a device address, so the
// looked-up pointer is what the kernels receive.
//
// Every call shares the one array and leaves its contents behind.  Nothing in
// it has to start at zero: the work planner rewrites every control word,
// counter and per-row entry at the start of each call before any other kernel
// reads them.  Two calls whose kernels overlap on the GPU (other streams,
// other host threads) race on the array.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PA_DECODE_NO_ALLOC_MAX_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

pa_status scratch_on_current_device(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_no_alloc(const void* q, const void* key_cache,
                                        const void* value_cache, const int32_t* block_tables,
                                        const int32_t* seq_lens, float scale, void* out,
                                        int32_t num_seqs, int32_t num_heads,
                                        int32_t max_blocks_per_seq, int32_t out_dtype,
                                        const pa_cache_desc* cache, int32_t* err_word,
                                        void* stream) {
  const size_t need =
      pa_decode_workspace_size(num_seqs, num_heads, max_blocks_per_seq, cache);
  if (need == 0 || num_seqs == 0) {
    // invalid arguments (or nothing to do): pa_decode reports which, before
    // it would ever look at a workspace
    return pa_decode(q, key_cache, value_cache, block_tables, seq_lens, scale, out, num_seqs,
                     num_heads, max_blocks_per_seq, out_dtype, cache, nullptr, 0, err_word,
                     stream);
  }
  if (need > static_cast<size_t>(PA_DECODE_NO_ALLOC_MAX_BYTES)) return PA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const pa_status st = scratch_on_current_device(&scratch);
  if (st != PA_OK) return st;
  return pa_decode(q, key_cache, value_cache, block_tables, seq_lens, scale, out, num_seqs,
                   num_heads, max_blocks_per_seq, out_dtype, cache, scratch,
                   static_cast<size_t>(PA_DECODE_NO_ALLOC_MAX_BYTES), err_word, stream);
}
