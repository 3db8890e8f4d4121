// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tiledattn.h"

namespace ta {

using PFN_encodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

// cuTensorMapEncodeTiled fetched through the runtime (no libcuda link).
PFN_encodeTiled get_encode_tiled();

// Tensor map over a bf16 array [slices, rows, d] (d contiguous, d = 64 or
// 128) whose box is a whole tile of 128 rows: 4-D {64, rows, d / 64, slices},
// coordinates (0, row, 0, slice), landing [64-column chunk][128 rows][128 B]
// with the 128-byte swizzle; rows past `rows` read as zero.
ta_status encode_rows_chunked(CUtensorMap* map, const void* base, int d, int rows, int slices);

// The same for a one-byte-per-element array (FP8 codes) [slices, rows, d],
// d = 128: {128, rows, 1, slices}, one 128-byte swizzle row per row.
ta_status encode_u8_rows_chunked(CUtensorMap* map, const void* base, int d, int rows, int slices);

// General bf16 tensor map (rank 2-5, 128-byte swizzle, zero fill out of
// bounds); strides_bytes has rank - 1 entries.
ta_status encode_bf16_tiled(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box);
// The same with the 32-byte swizzle (box rows of 32 bytes).
ta_status encode_bf16_tiled_sw32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                                 const uint64_t* strides_bytes, const uint32_t* box);

// Records a description of the last host-side failure of this thread
// (returned by ta_last_error) and returns `code`.
ta_status fail(ta_status code, const char* where, cudaError_t err = cudaSuccess);
ta_status fail_cu(ta_status code, const char* where, int cu_result);

// Device address of the library status word in the current context.
unsigned* device_status_ptr();

// Unique identifier (cuCtxGetId) of the CUDA context current on the calling
// thread.  Identifiers are never reused within a process, so a cache keyed by
// one never serves an address from a context that was destroyed (for example
// by cudaDeviceReset).  Returns false if no context is current or the driver
// entry points are unavailable.
bool current_context_id(unsigned long long* id);

// Small per-context cache of device addresses of __device__ variables (their
// host-side names are only stand-ins; the address comes from
// cudaGetSymbolAddress in the context that will use it).
class ContextAddressCache {
 public:
  bool find(unsigned long long ctx, void** out);
  void insert(unsigned long long ctx, void* p);

 private:
  static constexpr int kSlots = 16;
  std::mutex mu_;
  unsigned long long ids_[kSlots] = {};
  void* ptrs_[kSlots] = {};
  int next_ = 0;
};

// Raise a kernel's dynamic shared-memory limit once per device.
// `done` is the caller's per-kernel, per-device record.
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel kernel, int bytes, int (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // The flags may be read and set by several host threads: atomic accesses
  // (setting the attribute twice is harmless).
  if (dev >= 0 && dev < 64 && __atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) __atomic_store_n(&done[dev], 1, __ATOMIC_RELEASE);
  return e;
}

// Split-KV plan for paged decode (pure host arithmetic).
struct DecodePlan {
  int chunk_tokens;   // tokens staged per pipeline step (64)
  int split_pages;    // pages handled by one CTA
  int max_splits;     // ceil(max_pages / split_pages)
  size_t partial_o_offset, partial_lse_offset, bytes;
};
bool make_decode_plan(int num_seqs, int Hq, int Hkv, int d, int max_pages, int page_size, DecodePlan* plan);

ta_status launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream);

ta_status launch_prefill_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                             float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nkv,
                             float scale, int causal, cudaStream_t stream);

ta_status launch_paged_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                              const int32_t* seq_lens, int page_size, int num_seqs, int Hq, int Hkv, int d,
                              int max_pages, int num_pages_total, float scale, void* o, float* lse, void* workspace,
                              const DecodePlan& plan, cudaStream_t stream);

ta_status launch_gather_debug(const void* k_cache, const void* v_cache, const int32_t* block_table,
                              const int32_t* seq_lens, int seq, int hkv, int page_size, int Hkv, int d,
                              int max_pages, int num_pages_total, void* k_out, void* v_out, cudaStream_t stream);

ta_status launch_selftest_wait(unsigned limit_us, cudaStream_t stream);

ta_status launch_paged_prefill(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                               const int32_t* cu_seqlens, const int32_t* seq_lens, int page_size, int num_seqs,
                               int total_q, int max_q_len, int Hq, int Hkv, int d, int max_pages,
                               int num_pages_total, float scale, int causal, void* o, float* lse,
                               cudaStream_t stream);

ta_status launch_lse_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, int64_t rows,
                           int d, int first, cudaStream_t stream);
ta_status launch_lse_merge_finish(const float* acc_o, void* out, int64_t rows, int d, cudaStream_t stream);

size_t bwd_workspace_bytes(int B, int Hq, int Nq);
ta_status launch_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                          const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                          int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream);

}  // namespace ta
