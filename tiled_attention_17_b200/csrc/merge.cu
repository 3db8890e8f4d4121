// Log-sum-exp merge of partial attention results.
//
// Attention over a key set split into blocks can be computed block by block
// and the partial results combined exactly: each partial carries its output
// (normalised over its own keys) and the log of its normaliser, and
//
//   lse = log(e^lse_a + e^lse_b),  O = e^(lse_a - lse) O_a + e^(lse_b - lse) O_b
//
// (FlashAttention optimisation article, section 3.2.2: the online-softmax
// result does not depend on how the keys are blocked or ordered).  The ring
// schedule of the LLM-inference article (section 4.1) produces one such
// partial per hop; the accumulator is kept in fp32 between hops and converted
// to bf16 once at the end.  Both kernels are HBM-bound elementwise passes:
// one warp per row, 16-byte (fp32) and 8-byte (bf16) vector accesses.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tiledattn_internal.h"

namespace ta {
namespace {

// rows are processed one warp each; lane l owns columns [l * D/32, (l+1) * D/32)
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(float* __restrict__ acc_o, float* __restrict__ acc_lse,
                                                        const __nv_bfloat16* __restrict__ part_o,
                                                        const float* __restrict__ part_lse, int64_t rows,
                                                        int first) {
  constexpr int kPer = D / 32;   // 4 (d = 128) or 2 (d = 64)
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;   // whole warps leave together
  const float lp = part_lse[row];
  float* ao = acc_o + row * D + lane * kPer;
  const __nv_bfloat16* po = part_o + row * D + lane * kPer;
  float p[kPer];
  if constexpr (kPer == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(po);
    p[0] = __uint_as_float(w.x << 16);
    p[1] = __uint_as_float(w.x & 0xFFFF0000u);
    p[2] = __uint_as_float(w.y << 16);
    p[3] = __uint_as_float(w.y & 0xFFFF0000u);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(po);
    p[0] = __uint_as_float(w << 16);
    p[1] = __uint_as_float(w & 0xFFFF0000u);
  }
  float out[kPer];
  float lse_new;
  if (first) {
    lse_new = lp;
#pragma unroll
    for (int e = 0; e < kPer; ++e) out[e] = lp == -INFINITY ? 0.f : p[e];
  } else {
    const float la = acc_lse[row];
    const float m = fmaxf(la, lp);
    if (m == -INFINITY) {   // neither side has a visible key
      lse_new = -INFINITY;
#pragma unroll
      for (int e = 0; e < kPer; ++e) out[e] = 0.f;
    } else {
      const float wa = __expf(la - m), wp = __expf(lp - m);   // e^-inf = 0
      const float inv = 1.f / (wa + wp);
      float a[kPer];
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(ao);
        a[0] = v.x;
        a[1] = v.y;
        a[2] = v.z;
        a[3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(ao);
        a[0] = v.x;
        a[1] = v.y;
      }
#pragma unroll
      for (int e = 0; e < kPer; ++e) out[e] = (wa * a[e] + wp * p[e]) * inv;
      lse_new = m + __logf(wa + wp);
    }
  }
  if constexpr (kPer == 4)
    *reinterpret_cast<float4*>(ao) = make_float4(out[0], out[1], out[2], out[3]);
  else
    *reinterpret_cast<float2*>(ao) = make_float2(out[0], out[1]);
  if (lane == 0) acc_lse[row] = lse_new;
}

template <int D>
__global__ void __launch_bounds__(256) lse_merge_finish_kernel(const float* __restrict__ acc_o,
                                                               __nv_bfloat16* __restrict__ out, int64_t n4) {
  // four values per thread (D is a multiple of 4)
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(acc_o)[i];
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  reinterpret_cast<uint2*>(out)[i] = w;
}

}  // namespace

ta_status launch_lse_merge(float* acc_o, float* acc_lse, const void* part_o, const float* part_lse, int64_t rows,
                           int d, int first, cudaStream_t stream) {
  const int64_t threads = rows * 32;
  const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
  if (d == 128)
    lse_merge_kernel<128><<<grid, 256, 0, stream>>>(acc_o, acc_lse, static_cast<const __nv_bfloat16*>(part_o),
                                                    part_lse, rows, first);
  else
    lse_merge_kernel<64><<<grid, 256, 0, stream>>>(acc_o, acc_lse, static_cast<const __nv_bfloat16*>(part_o),
                                                   part_lse, rows, first);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "attn_lse_merge: launch", e);
}

ta_status launch_lse_merge_finish(const float* acc_o, void* out, int64_t rows, int d, cudaStream_t stream) {
  const int64_t n4 = rows * d / 4;
  const unsigned grid = static_cast<unsigned>((n4 + 255) / 256);
  if (d == 128)
    lse_merge_finish_kernel<128><<<grid, 256, 0, stream>>>(acc_o, static_cast<__nv_bfloat16*>(out), n4);
  else
    lse_merge_finish_kernel<64><<<grid, 256, 0, stream>>>(acc_o, static_cast<__nv_bfloat16*>(out), n4);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "attn_lse_merge_finish: launch", e);
}

}  // namespace ta
