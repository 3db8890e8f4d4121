// C ABI of libtiledattn.so: host-side argument validation, the library status
// word, and dispatch to the kernels.  Declarations and the contract of every
// entry point are in include/tiledattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "ptx.cuh"
#include "tiledattn_internal.h"

namespace ta {

static_assert(kDevTimeout == TA_DEV_TIMEOUT && kDevBadBlockTable == TA_DEV_BAD_BLOCK_TABLE &&
                  kDevBadSeqLen == TA_DEV_BAD_SEQ_LEN,
              "device status bits");

// One status word per device (a __device__ variable exists once per device
// the library is loaded on).  Bits: TA_DEV_*.
__device__ unsigned g_status_word;

using PFN_ctxGetCurrent = CUresult (*)(CUcontext*);
using PFN_ctxGetId = CUresult (*)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id) {
  static PFN_ctxGetCurrent get_current = nullptr;
  static PFN_ctxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctxGetId>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

bool ContextAddressCache::find(unsigned long long ctx, void** out) {
  std::lock_guard<std::mutex> g(mu_);
  for (int i = 0; i < kSlots; ++i)
    if (ptrs_[i] && ids_[i] == ctx) {
      *out = ptrs_[i];
      return true;
    }
  return false;
}

void ContextAddressCache::insert(unsigned long long ctx, void* p) {
  std::lock_guard<std::mutex> g(mu_);
  ids_[next_] = ctx;
  ptrs_[next_] = p;
  next_ = (next_ + 1) % kSlots;
}

unsigned* device_status_ptr() {
  static ContextAddressCache cache;
  unsigned long long ctx = 0;
  void* p = nullptr;
  if (current_context_id(&ctx) && cache.find(ctx, &p)) return static_cast<unsigned*>(p);
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess || p == nullptr) return nullptr;
  // the lookup made the device's primary context current if none was
  if (current_context_id(&ctx)) cache.insert(ctx, p);
  return static_cast<unsigned*>(p);
}

PFN_encodeTiled get_encode_tiled() {
  static PFN_encodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(p);
  });
  return fn;
}

static ta_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank,
                              const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  PFN_encodeTiled enc = get_encode_tiled();
  if (!enc) return fail(TA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = enc(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d,
                   st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TA_OK : fail_cu(TA_ERR_CUDA, "cuTensorMapEncodeTiled", static_cast<int>(r));
}

ta_status encode_bf16_tiled(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                            const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

ta_status encode_bf16_tiled_sw32(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                                 const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                      CU_TENSOR_MAP_SWIZZLE_32B);
}

// Tiles of 128 rows of a [slices, rows, d] tensor, each in ONE copy: the map
// is 4-D {one 128-byte chunk of columns, rows, d / chunk, slices} with the
// chunk stride of 128 bytes, so a box {chunk, 128, d / chunk, 1} lands a tile
// as [chunk][128 rows][128 B], the 128-byte-swizzle layout of every chunk.
// (A copy has a fixed cost in the SM's copy engine.  For these 16 KB chunks it
// is small beside the bytes: one copy per tile times the same as one per
// chunk.  For page-sized copies it is not; see the paged prefill.)
ta_status encode_u8_rows_chunked(CUtensorMap* map, const void* base, int d, int rows, int slices) {
  const uint64_t dims[4] = {128, static_cast<uint64_t>(rows), static_cast<uint64_t>(d / 128),
                            static_cast<uint64_t>(slices)};
  const uint64_t strides[3] = {static_cast<uint64_t>(d), 128, static_cast<uint64_t>(rows) * d};
  const uint32_t box[4] = {128, 128, static_cast<uint32_t>(d / 128), 1};
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 4, dims, strides, box);
}

ta_status encode_rows_chunked(CUtensorMap* map, const void* base, int d, int rows, int slices) {
  const uint64_t dims[4] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(d / 64),
                            static_cast<uint64_t>(slices)};
  const uint64_t strides[3] = {static_cast<uint64_t>(d) * 2, 128, static_cast<uint64_t>(rows) * d * 2};
  const uint32_t box[4] = {64, 128, static_cast<uint32_t>(d / 64), 1};
  return encode_bf16_tiled(map, base, 4, dims, strides, box);
}

static thread_local char g_last_error[256] = "";

ta_status fail(ta_status code, const char* where, cudaError_t err) {
  if (err != cudaSuccess)
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(err), cudaGetErrorString(err));
  else
    snprintf(g_last_error, sizeof g_last_error, "%s", where);
  return code;
}

ta_status fail_cu(ta_status code, const char* where, int cu_result) {
  snprintf(g_last_error, sizeof g_last_error, "%s: CUresult %d", where, cu_result);
  return code;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace ta

using namespace ta;

// The FMA-pipe exponential of the FP8 softmax, evaluated on its own (the
// ta_exp2_poly_debug test export): pairs, as the softmax evaluates them.
__global__ void __launch_bounds__(256) exp2_poly_debug_kernel(const float* __restrict__ x, float* __restrict__ y,
                                                              long long n) {
  const long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float2 r = exp2_poly2(make_float2(x[i], two ? x[i + 1] : 0.f));
  y[i] = r.x;
  if (two) y[i + 1] = r.y;
}

extern "C" {

const char* ta_status_string(ta_status s) {
  switch (s) {
    case TA_OK: return "TA_OK";
    case TA_ERR_INVALID_ARG: return "TA_ERR_INVALID_ARG";
    case TA_ERR_UNSUPPORTED: return "TA_ERR_UNSUPPORTED";
    case TA_ERR_CUDA: return "TA_ERR_CUDA";
    case TA_ERR_BAD_BLOCK_TABLE: return "TA_ERR_BAD_BLOCK_TABLE";
    case TA_ERR_DEVICE_TIMEOUT: return "TA_ERR_DEVICE_TIMEOUT";
  }
  return "TA_ERR_UNKNOWN";
}

int ta_version(void) { return 10000; }

const char* ta_last_error(void) { return g_last_error; }

ta_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                   int Nkv, int d, float scale, int causal, ta_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0) return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return TA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  // sizes the kernels index with 32-bit coordinates
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || Nq > (1 << 30) || Nkv > (1 << 30)) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq * Nq == 0) return TA_OK;
  if (!q || !o || (Nkv > 0 && (!k || !v))) return TA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return TA_ERR_INVALID_ARG;
  const long long pairs = (static_cast<long long>(Nq) + 255) / 256;
  if (pairs * B * Hq > INT32_MAX) return TA_ERR_UNSUPPORTED;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, reinterpret_cast<cudaStream_t>(stream));
}

ta_status attn_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                       float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                       float scale, int causal, ta_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0) return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return TA_ERR_UNSUPPORTED;
  for (float ds : {q_descale, k_descale, v_descale})
    if (!std::isfinite(ds) || ds <= 0.f) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(scale * q_descale * k_descale)) return TA_ERR_UNSUPPORTED;
  if (d != 128) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || Nq > (1 << 30) || Nkv > (1 << 30)) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq * Nq == 0) return TA_OK;
  if (!q || !o || (Nkv > 0 && (!k || !v))) return TA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return TA_ERR_INVALID_ARG;
  const long long pairs = (static_cast<long long>(Nq) + 255) / 256;
  if (pairs * B * Hq > INT32_MAX) return TA_ERR_UNSUPPORTED;
  return launch_prefill_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal,
                            reinterpret_cast<cudaStream_t>(stream));
}

ta_status attn_paged_prefill(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                             const int32_t* cu_seqlens, const int32_t* seq_lens, int page_size, int num_seqs,
                             int total_q, int max_q_len, int Hq, int Hkv, int d, int max_pages, int num_pages_total,
                             float scale, int causal, void* o, float* lse, ta_stream_t stream) {
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || page_size <= 0 ||
      max_pages <= 0 || num_pages_total <= 0)
    return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return TA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  if (page_size != 8 && page_size != 16 && page_size != 32 && page_size != 64) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_pages) * page_size > (1 << 30) || Hq > 65535) return TA_ERR_UNSUPPORTED;
  // the K copies address a (page, KV head) block by one 32-bit coordinate
  if (static_cast<long long>(num_pages_total) * Hkv > INT32_MAX) return TA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return TA_OK;
  const long long pairs = (static_cast<long long>(max_q_len) + 255) / 256;
  if (pairs * num_seqs * Hq > INT32_MAX) return TA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !block_table || !cu_seqlens || !seq_lens || !o) return TA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return TA_ERR_INVALID_ARG;
  return launch_paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, page_size, num_seqs, total_q,
                              max_q_len, Hq, Hkv, d, max_pages, num_pages_total, scale, causal, o, lse,
                              reinterpret_cast<cudaStream_t>(stream));
}

ta_status attn_lse_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, int64_t rows, int d,
                         int first, ta_stream_t stream) {
  if (rows < 0 || d <= 0 || (first != 0 && first != 1)) return TA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  if (rows > (int64_t(1) << 33)) return TA_ERR_UNSUPPORTED;   // grid of rows / 8 blocks
  if (rows == 0) return TA_OK;
  if (!acc_o || !acc_lse || !part_o || !part_lse) return TA_ERR_INVALID_ARG;
  if (!aligned16(acc_o) || (reinterpret_cast<uintptr_t>(part_o) & 7u) || (reinterpret_cast<uintptr_t>(acc_lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(part_lse) & 3u))
    return TA_ERR_INVALID_ARG;
  return launch_lse_merge(acc_o, acc_lse, part_o, part_lse, rows, d, first, reinterpret_cast<cudaStream_t>(stream));
}

ta_status attn_lse_merge_finish(const float* acc_o, void* out, int64_t rows, int d, ta_stream_t stream) {
  if (rows < 0 || d <= 0) return TA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  if (rows > (int64_t(1) << 33)) return TA_ERR_UNSUPPORTED;   // grid of rows / 8 blocks
  if (rows == 0) return TA_OK;
  if (!acc_o || !out || !aligned16(acc_o) || (reinterpret_cast<uintptr_t>(out) & 7u)) return TA_ERR_INVALID_ARG;
  return launch_lse_merge_finish(acc_o, out, rows, d, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_bwd_workspace_size(int B, int Hq, int Nq) {
  if (B < 0 || Hq <= 0 || Nq < 0) return 0;
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || Nq > (1 << 30)) return 0;
  return bwd_workspace_bytes(B, Hq, Nq);
}

ta_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                   int Nq, int Nkv, int d, float scale, int causal, ta_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nkv < 0 || d <= 0) return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return TA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return TA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq > INT32_MAX / 2 || Nq > (1 << 30) || Nkv > (1 << 30)) return TA_ERR_UNSUPPORTED;
  const long long q_tiles = (static_cast<long long>(Nq) + 127) / 128, k_tiles = (static_cast<long long>(Nkv) + 127) / 128;
  if (q_tiles * B * Hq > INT32_MAX || k_tiles * B * Hkv > INT32_MAX) return TA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t q_bytes = static_cast<size_t>(B) * Hq * Nq * d * 2;
  const size_t kv_bytes = static_cast<size_t>(B) * Hkv * Nkv * d * 2;
  if (q_bytes == 0 && kv_bytes == 0) return TA_OK;
  if ((q_bytes && (!q || !o || !dout || !lse || !dq)) || (kv_bytes && (!k || !v || !dk || !dv)))
    return TA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return TA_ERR_INVALID_ARG;
  // no queries: no gradient reaches K or V; no keys: none reaches Q
  if (q_bytes == 0 || kv_bytes == 0) {
    cudaError_t e = cudaSuccess;
    if (kv_bytes) {
      if ((e = cudaMemsetAsync(dk, 0, kv_bytes, st)) == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, st);
    }
    if (q_bytes && e == cudaSuccess) e = cudaMemsetAsync(dq, 0, q_bytes, st);
    return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "attn_bwd: zero fill", e);
  }
  const size_t need = bwd_workspace_bytes(B, Hq, Nq);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) {
    char msg[160];
    snprintf(msg, sizeof msg, "attn_bwd: workspace needs %zu bytes, 256-byte aligned", need);
    return fail(TA_ERR_INVALID_ARG, msg);
  }
  return launch_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nkv, d, scale, causal, st);
}

size_t attn_paged_decode_workspace_size(int num_seqs, int Hq, int Hkv, int d, int max_pages, int page_size) {
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv) return 0;
  DecodePlan plan;
  if (!make_decode_plan(num_seqs, Hq, Hkv, d, max_pages, page_size, &plan)) return 0;
  return plan.bytes;
}

static ta_status validate_decode_shape(int page_size, int num_seqs, int Hq, int Hkv, int d, int max_pages,
                                       int num_pages_total) {
  if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || max_pages <= 0 || num_pages_total <= 0 || page_size <= 0)
    return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return TA_ERR_UNSUPPORTED;
  if (page_size != 8 && page_size != 16 && page_size != 32 && page_size != 64) return TA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return TA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || Hkv > 65535) return TA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_pages) * page_size > INT32_MAX) return TA_ERR_UNSUPPORTED;
  return TA_OK;
}

ta_status attn_paged_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                            const int32_t* seq_lens, int page_size, int num_seqs, int Hq, int Hkv, int d,
                            int max_pages, int num_pages_total, float scale, void* o, float* lse, void* workspace,
                            size_t workspace_bytes, ta_stream_t stream) {
  ta_status st = validate_decode_shape(page_size, num_seqs, Hq, Hkv, d, max_pages, num_pages_total);
  if (st != TA_OK) return st;
  if (!std::isfinite(scale) || scale < 0.f) return TA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return TA_OK;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o || !workspace) return TA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return TA_ERR_INVALID_ARG;
  DecodePlan plan;
  if (!make_decode_plan(num_seqs, Hq, Hkv, d, max_pages, page_size, &plan)) return TA_ERR_UNSUPPORTED;
  if (workspace_bytes < plan.bytes) return TA_ERR_INVALID_ARG;
  return launch_paged_decode(q, k_cache, v_cache, block_table, seq_lens, page_size, num_seqs, Hq, Hkv, d, max_pages,
                             num_pages_total, scale, o, lse, workspace, plan, reinterpret_cast<cudaStream_t>(stream));
}

ta_status attn_paged_decode_check(const void* workspace, unsigned* flags, ta_stream_t stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return TA_ERR_INVALID_ARG;
  unsigned w = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess) return TA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TA_ERR_CUDA;
  if (flags) *flags = w;
  if (w & TA_DEV_TIMEOUT) return TA_ERR_DEVICE_TIMEOUT;
  if (w & (TA_DEV_BAD_BLOCK_TABLE | TA_DEV_BAD_SEQ_LEN)) return TA_ERR_BAD_BLOCK_TABLE;
  return TA_OK;
}

ta_status attn_paged_gather_debug(const void* k_cache, const void* v_cache, const int32_t* block_table,
                                  const int32_t* seq_lens, int seq, int hkv, int page_size, int Hkv, int d,
                                  int max_pages, int num_pages_total, void* k_out, void* v_out, ta_stream_t stream) {
  ta_status st = validate_decode_shape(page_size, seq + 1, Hkv, Hkv, d, max_pages, num_pages_total);
  if (st != TA_OK) return st;
  if (seq < 0 || hkv < 0 || hkv >= Hkv) return TA_ERR_INVALID_ARG;
  if (!k_cache || !v_cache || !block_table || !seq_lens || !k_out || !v_out) return TA_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_out) || !aligned16(v_out) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return TA_ERR_INVALID_ARG;
  return launch_gather_debug(k_cache, v_cache, block_table, seq_lens, seq, hkv, page_size, Hkv, d, max_pages,
                             num_pages_total, k_out, v_out, reinterpret_cast<cudaStream_t>(stream));
}

ta_status ta_device_status(unsigned* flags, int reset) {
  unsigned* p = device_status_ptr();
  if (!p) return TA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return TA_ERR_CUDA;
  unsigned w = 0;
  if (cudaMemcpy(&w, p, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return TA_ERR_CUDA;
  if (reset && cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return TA_ERR_CUDA;
  if (flags) *flags = w;
  if (w & TA_DEV_TIMEOUT) return TA_ERR_DEVICE_TIMEOUT;
  if (w & (TA_DEV_BAD_BLOCK_TABLE | TA_DEV_BAD_SEQ_LEN)) return TA_ERR_BAD_BLOCK_TABLE;
  return TA_OK;
}

ta_status ta_selftest_bounded_wait(unsigned limit_us, ta_stream_t stream) {
  if (limit_us == 0 || limit_us > 1000000u) return TA_ERR_INVALID_ARG;
  return launch_selftest_wait(limit_us, reinterpret_cast<cudaStream_t>(stream));
}

ta_status ta_exp2_poly_debug(const float* x, float* y, int64_t n, ta_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y)) || (reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u))
    return TA_ERR_INVALID_ARG;
  if (n == 0) return TA_OK;
  const long long pairs = (n + 1) / 2;
  exp2_poly_debug_kernel<<<static_cast<unsigned>((pairs + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, y, static_cast<long long>(n));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "ta_exp2_poly_debug: launch", e);
}

}  // extern "C"
