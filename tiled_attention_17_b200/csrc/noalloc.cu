// Paged decode for callers that cannot allocate device memory.
//
// attn_paged_decode needs a caller-provided workspace for its split-KV
// partials.  Some callers have no way to obtain one: a plugin running inside a
// host framework that owns all device memory and hands the plugin only its
// input and output buffers, or code on a latency-critical path where the
// implicit device-wide synchronisation of cudaMalloc/cudaFree is not
// acceptable.  attn_paged_decode_noalloc serves them with a fixed scratch area
// that lives in this library's own device memory instead.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes.  In
// host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress once per CUDA context (on
// each device, with that device current) and cached.  The call then forwards
// to attn_paged_decode with that address as the workspace, so the kernels,
// validation and launch path are exactly those of attn_paged_decode.
#include <cuda_runtime.h>

#include <cstdio>

#include "tiledattn_internal.h"

namespace ta {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB

// Shared by every call on a device; holds the last call's partials and status
// word until the next call overwrites them.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the calling thread's current
// context.  The host-side name g_noalloc_scratch is only a stand-in, so the
// address is looked up with cudaGetSymbolAddress, with the device (and the
// context that will run the kernels) current, on the first call in each
// context, and cached under that context's unique identifier.  A context
// created later (after cudaDeviceReset, or one the caller makes current) gets
// a lookup of its own, never a stale address.
static ta_status noalloc_scratch(void** out) {
  static ContextAddressCache cache;
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) && cache.find(ctx, out)) return TA_OK;
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return fail(TA_ERR_CUDA, "attn_paged_decode_noalloc: cudaGetSymbolAddress of the scratch array", e);
  // the lookup made the device's primary context current if none was
  if (current_context_id(&ctx)) cache.insert(ctx, p);
  *out = p;
  return TA_OK;
}

}  // namespace ta

extern "C" ta_status attn_paged_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                               const int32_t* block_table, const int32_t* seq_lens, int page_size,
                                               int num_seqs, int Hq, int Hkv, int d, int max_pages,
                                               int num_pages_total, float scale, void* o, float* lse,
                                               ta_stream_t stream) {
  using namespace ta;
  const size_t need = attn_paged_decode_workspace_size(num_seqs, Hq, Hkv, d, max_pages, page_size);
  if (need > kNoAllocScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof msg,
             "attn_paged_decode_noalloc: these sizes need %zu bytes of scratch, more than the %zu built in",
             need, kNoAllocScratchBytes);
    return fail(TA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  ta_status st = noalloc_scratch(&scratch);
  if (st != TA_OK) return st;
  // Invalid sizes (need == 0) are rejected by attn_paged_decode's own checks.
  return attn_paged_decode(q, k_cache, v_cache, block_table, seq_lens, page_size, num_seqs, Hq, Hkv, d, max_pages,
                           num_pages_total, scale, o, lse, scratch, kNoAllocScratchBytes, stream);
}
