// paged_attention_decode_noalloc: the paged decode call for callers that
// cannot allocate device memory.
//
// The regular decode call takes a caller-owned workspace for the split-KV
// partials. Some callers cannot provide one: a runtime that has handed all
// device memory to its own pool and forbids allocations outside it, a plain
// C or embedded host without a device allocator at hand, or a latency-bound
// loop that cannot afford cudaMalloc (which may synchronise the device). This
// variant runs the same kernels with the scratch in a fixed array that lives
// in this library's device image instead.
//
// Facts a caller must know:
//  * The scratch is a file-scope __device__ array of kNoAllocScratchBytes
//    (8 MiB). Every GPU on which this library's kernels are loaded holds it
//    until the process exits.
//  * Its device address is looked up once per device, with that device
//    current, by the first call made on that device (cudaGetSymbolAddress);
//    make that first call before any stream capture begins.
//  * All calls share the one array and it keeps the last call's contents.
//    Nothing in it needs to start at zero: every word the merge step reads
//    is written earlier by the same call. Calls that overlap on the GPU (on
//    different streams, or from different threads without ordering) race
//    on the scratch and give wrong results; order them on one stream.
//  * A problem whose scratch need exceeds the array is rejected with
//    PKV_ERR_WORKSPACE_TOO_SMALL before anything is launched.
//  * The call allocates and frees nothing (no cudaMalloc, no cudaFree, no
//    allocating library routine).
#include <mutex>

#include "pkv_common.cuh"
#include "pkv_internal.h"

namespace pkv {

constexpr size_t kNoAllocScratchBytes = size_t(PKV_NOALLOC_SCRATCH_BYTES);

// The scratch itself. In host code this name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch on the current device (looked up once).
int scratch_on_current_device(void** addr) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return fail(PKV_ERR_CUDA, "paged_attention_decode_noalloc: cudaGetDevice: %s",
                cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PKV_ERR_UNSUPPORTED, "paged_attention_decode_noalloc: device index %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(PKV_ERR_CUDA, "paged_attention_decode_noalloc: cudaGetSymbolAddress: %s",
                  cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" PKV_API int paged_attention_decode_noalloc(
    const void* q, const void* k_cache, const void* v_cache, pkv_cache_desc cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
    int32_t batch, int32_t num_q_heads, float scale, pkv_mask_mod mask, void* out, float* lse,
    int32_t* dbg_err, void* stream) {
  using namespace pkv;
  if (batch < 0) {
    clear_last_error();
    return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode_noalloc: bad batch");
  }
  const size_t need = paged_attention_decode_workspace_size(batch, num_q_heads, cache);
  if (need > kNoAllocScratchBytes)
    return fail(PKV_ERR_WORKSPACE_TOO_SMALL,
                "paged_attention_decode_noalloc: this problem needs %zu bytes of scratch but the "
                "built-in scratch holds %zu; use paged_attention_decode with a workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (need > 0) {
    if (int st = scratch_on_current_device(&scratch)) return st;
  }
  return paged_attention_decode(q, k_cache, v_cache, cache, block_tables, max_blocks_per_seq,
                                seq_lens, batch, num_q_heads, scale, mask, out, lse, scratch,
                                need > 0 ? kNoAllocScratchBytes : 0, dbg_err, stream);
}
