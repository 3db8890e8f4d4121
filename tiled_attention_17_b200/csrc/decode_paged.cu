// Split-KV paged decode for sm_100a: one query token per sequence against a
// paged KV cache, followed by a log-sum-exp combine of the splits.
//
// The pool holds fixed-size pages [num_pages_total, Hkv, page_size, d]; a
// sequence's pages are listed in its block-table row (PagedAttention,
// GPU-optimisation tag page).  The gather follows the paged gather article,
// section 2:
//   2.1  a CTA stages the scattered pages of its range into shared memory;
//        here each (page, KV head) is one contiguous page_size*d*2-byte span,
//        so one TMA bulk copy moves it and every byte read is used;
//   2.3  the split's block-table entries are loaded once, before the gather
//        loop, into a shared-memory table that every copy reads (index
//        prefetch);
//   2.4  the gather is fused with the dot products q.k, the online softmax
//        and the weighted sum of V; nothing gathered is written back.
// Splits are merged by their log-sum-exp, which is exact because the online
// softmax result does not depend on how the keys are grouped (FlashAttention
// optimisation article, section 3.2.2).
//
// Kernel 1 (decode_split_kernel): one CTA per (split, KV head, sequence);
//   the G = Hq/Hkv query heads of the KV head are handled together so every
//   K/V byte is read from HBM once.  A 3-stage ring of 64-token chunks keeps
//   up to 96 KB per CTA in flight.  Per chunk:
//     A) scores: 16 lanes cover one 256-byte K row with 16-byte shared loads,
//        dot with the G query slices held in registers, reduce across lanes;
//     B) online softmax per head (one warp per head): chunk max, rescale
//        factor e^(m_old - m_new), probabilities, running sum;
//     C) O_partial = alpha * O_partial + sum_t p_t v_t.
// Kernel 2 (decode_combine_kernel): one CTA per (query head, sequence).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "tiledattn_internal.h"

namespace ta {

constexpr int kChunkTokens = 64;           // tokens staged per pipeline step
constexpr int kDecStages = 3;              // ring depth
constexpr int kConsumerWarps = 8;          // each owns 8 rows of every chunk
constexpr int kRowsPerWarp = kChunkTokens / kConsumerWarps;
constexpr int kSplitThreads = 32 * (kConsumerWarps + 1);   // + one TMA producer warp
constexpr int kGatherThreads = 128;        // gather-debug kernel
constexpr int kMaxG = 8;
// Tokens per split of a sequence's keys.  2048 measured 4% faster than 1024
// on the 64-sequence benchmark batch (half the CTAs, so half their fixed
// cost: table staging, first-chunk latency, partial write) and equal to 4096.
constexpr int kSplitTokens = 2048;
constexpr int kMaxSplitPages = kSplitTokens / 8;   // block-table entries one split stages (8-token pages)

template <int D>
struct DecodeLayout {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunkBytes = kChunkTokens * kRowBytes;
  static constexpr int kStageBytes = 2 * kChunkBytes;   // K chunk then V chunk
  static constexpr int kRing = kDecStages * kStageBytes;
  static constexpr int kLanesPerRow = D / 8;            // 16-byte slices per row
  static constexpr int kSegs = 32 / kLanesPerRow;       // rows a warp covers per pass
  static constexpr int kPasses = kRowsPerWarp / kSegs;
  // end-of-split merge of the per-segment states (reuses the ring's space)
  static constexpr int kStates = kConsumerWarps * kSegs;
  template <int G>
  static constexpr int merge_bytes() { return kStates * G * (D + 2) * 4; }
  static constexpr int kArea = kRing > kStates * kMaxG * (D + 2) * 4 ? kRing : kStates * kMaxG * (D + 2) * 4;
  static constexpr int kBar = kArea;                    // full[S], empty[S]
  static constexpr int kAbort = kBar + 2 * kDecStages * 8;
  static constexpr int kTable = kAbort + 16;            // the split's block-table entries
  static constexpr int kBytes = kTable + kMaxSplitPages * 4;
};

struct DecodeArgs {
  const __nv_bfloat16* q;
  const uint8_t* k_cache;
  const uint8_t* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int page_size, num_seqs, Hq, Hkv, max_pages, num_pages_total;
  int split_pages, max_splits;
  float scale, scale_log2;
  float* part_o;
  float* part_lse;
  unsigned* status;
};

__device__ __forceinline__ int clamp_len(int len, const DecodeArgs& a) {
  const int cap = a.max_pages * a.page_size;
  return len < 0 ? 0 : (len > cap ? cap : len);
}

// ---------------------------------------------------------------------------
// The page gather, shared by both split kernels and the gather-debug export
// (so the export checks the addressing the decode kernels run).
// ---------------------------------------------------------------------------
// Index prefetch (paged gather article, section 2.3): the block-table entries
// of one split's pages are loaded once into the shared-memory table `tbl` and
// checked there; every copy of the split then reads its page id from the
// table.  Entries outside [0, num_pages_total) are replaced by page 0 (never
// dereferenced) and flagged.  Thread i of the caller's `count` participating
// threads loads entries i, i + count, ...; the caller synchronises before the
// table is read.
__device__ __forceinline__ void load_split_table(const DecodeArgs& a, int seq, int split_first_page, int npages,
                                                 int* tbl, int i0, int count) {
  const int32_t* row = a.block_table + static_cast<size_t>(seq) * a.max_pages + split_first_page;
  for (int i = i0; i < npages; i += count) {
    int pg = __ldg(row + i);
    if (pg < 0 || pg >= a.num_pages_total) {
      atomicOr(a.status, kDevBadBlockTable);
      pg = 0;
    }
    tbl[i] = pg;
  }
}

// The copies of one chunk (paged gather article, section 2.1): pages
// [first, first + npg) of the split's table, each (page, KV head) one
// contiguous page_size * D * 2-byte span, land back to back in dstK / dstV
// (so chunk row r is token r of the chunk); `bar` is armed with their byte
// count.  Warp-wide: every lane of the calling warp must call it; lane i < npg
// copies page first + i.
template <int D>
__device__ __forceinline__ void gather_chunk(const DecodeArgs& a, int hkv, const int* tbl, int first, int npg,
                                             uint32_t dstK, uint32_t dstV, uint32_t bar) {
  const int lane = threadIdx.x & 31;
  const uint32_t page_bytes = static_cast<uint32_t>(a.page_size) * D * 2;
  if (lane == 0) mbar_arrive_expect_tx(bar, 2u * npg * page_bytes);
  __syncwarp();
  if (lane < npg) {
    const size_t off = (static_cast<size_t>(tbl[first + lane]) * a.Hkv + hkv) * page_bytes;
    bulk_load(dstK + lane * page_bytes, a.k_cache + off, page_bytes, bar);
    bulk_load(dstV + lane * page_bytes, a.v_cache + off, page_bytes, bar);
  }
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Sum each head's partial dot product over the LPR lanes that share a row, so
// that every lane of the row segment ends with all G totals.  For G = 4 a
// reduce-scatter followed by an all-gather needs 8 shuffles instead of 16.
template <int G, int LPR>
__device__ __forceinline__ void segment_allreduce(float (&v)[G], uint32_t mask, int lane_r) {
  if constexpr (G == 4) {
    constexpr int H1 = LPR / 2, H2 = LPR / 4;
    const bool b1 = lane_r & H1, b2 = lane_r & H2;
    float k0 = b1 ? v[2] : v[0], k1 = b1 ? v[3] : v[1];
    const float s0 = b1 ? v[0] : v[2], s1 = b1 ? v[1] : v[3];
    k0 += __shfl_xor_sync(mask, s0, H1);
    k1 += __shfl_xor_sync(mask, s1, H1);
    float x = b2 ? k1 : k0;
    x += __shfl_xor_sync(mask, b2 ? k0 : k1, H2);
#pragma unroll
    for (int o = H2 / 2; o >= 1; o >>= 1) x += __shfl_xor_sync(mask, x, o);
    // x = total of head (b1 ? 2 : 0) + (b2 ? 1 : 0); gather the other three
    const float xo = __shfl_xor_sync(mask, x, H2);
    const float lo = b2 ? xo : x, hi = b2 ? x : xo;
    const float lo2 = __shfl_xor_sync(mask, lo, H1), hi2 = __shfl_xor_sync(mask, hi, H1);
    v[0] = b1 ? lo2 : lo;
    v[1] = b1 ? hi2 : hi;
    v[2] = b1 ? lo : lo2;
    v[3] = b1 ? hi : hi2;
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int o = LPR / 2; o >= 1; o >>= 1) v[g] += __shfl_xor_sync(mask, v[g], o);
  }
}

constexpr float kDecRescaleLog2 = 8.0f;   // keep a stale max until it is exceeded by 2^8

template <int D, int G>
__global__ void __launch_bounds__(kSplitThreads, (G <= 4 ? 2 : 1)) decode_split_kernel(const DecodeArgs a) {
  using L = DecodeLayout<D>;
  constexpr int LPR = L::kLanesPerRow;
  constexpr int SEGS = L::kSegs;
  constexpr int PASSES = L::kPasses;
  static_assert(L::template merge_bytes<G>() <= L::kArea, "merge area fits");
  extern __shared__ __align__(1024) uint8_t smem[];

  const int split = blockIdx.x, hkv = blockIdx.y, seq = blockIdx.z;
  const int raw_len = __ldg(a.seq_lens + seq);
  const int len = clamp_len(raw_len, a);
  if (raw_len != len && split == 0 && hkv == 0 && threadIdx.x == 0) atomicOr(a.status, kDevBadSeqLen);
  const int split_tokens = a.split_pages * a.page_size;
  const int t_begin = split * split_tokens;
  if (t_begin >= len) return;  // CTA-uniform: nothing in this split
  const int t_end = min(len, t_begin + split_tokens);
  const int n_chunks = (t_end - t_begin + kChunkTokens - 1) / kChunkTokens;
  const int split_first_page = split * a.split_pages;
  const int split_npages = (t_end - t_begin + a.page_size - 1) / a.page_size;
  const int pages_per_chunk = kChunkTokens / a.page_size;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  auto FULL = [&](int s) { return sbase + L::kBar + 8u * s; };
  auto EMPTY = [&](int s) { return sbase + L::kBar + 8u * (kDecStages + s); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // per-segment online-softmax state (a segment = the LPR lanes of one row)
  const int lane_r = lane % LPR;   // 16-byte slice of a row
  const int seg = lane / LPR;
  float m[G], l[G];
  float2 acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = make_float2(0.f, 0.f);
  }

  if (warp == kConsumerWarps) {
    // ======================= producer warp =======================
    int* tbl = reinterpret_cast<int*>(smem + L::kTable);
    load_split_table(a, seq, split_first_page, split_npages, tbl, lane, 32);   // index prefetch
    __syncwarp();
    int c = 0;
    for (; c < n_chunks; ++c) {
      const int stage = c % kDecStages;
      bool ok = mbar_wait(EMPTY(stage), ((c / kDecStages) & 1u) ^ 1u, a.status, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int first = c * pages_per_chunk;
      const int npg = min(pages_per_chunk, split_npages - first);
      const uint32_t st = sbase + stage * L::kStageBytes;
      gather_chunk<D>(a, hkv, tbl, first, npg, st, st + L::kChunkBytes, FULL(stage));
    }
    // drain: no copy into this CTA's shared memory may be in flight at exit
    if (lane == 0)
      for (int cc = max(0, c - kDecStages); cc < c; ++cc)
        mbar_wait(FULL(cc % kDecStages), (cc / kDecStages) & 1u, nullptr, nullptr, kWaitLimitNs);
  } else {
    // ======================= consumer warps =======================
    const uint32_t seg_mask = (LPR == 32 ? 0xffffffffu : ((1u << LPR) - 1u) << (seg * LPR));
    float2 qf[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(a.q + (static_cast<size_t>(seq) * a.Hq + hkv * G + g) * D) +
                            lane_r);
      qf[g][0] = bf16x2_to_f2(u.x);
      qf[g][1] = bf16x2_to_f2(u.y);
      qf[g][2] = bf16x2_to_f2(u.z);
      qf[g][3] = bf16x2_to_f2(u.w);
    }
    const float c2 = a.scale_log2;
    const float thr = c2 > 0.f ? kDecRescaleLog2 / c2 : INFINITY;   // raw-score margin for a stale max

    for (int c = 0; c < n_chunks; ++c) {
      const int stage = c % kDecStages;
      bool ok = mbar_wait(FULL(stage), (c / kDecStages) & 1u, a.status, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* sK = smem + stage * L::kStageBytes;
      const uint8_t* sV = sK + L::kChunkBytes;
      const int valid = min(kChunkTokens, t_end - (t_begin + c * kChunkTokens));
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        const int row0 = warp * kRowsPerWarp + p * SEGS;
        if (row0 >= valid) break;                          // warp-uniform
        const int row = row0 + seg;
        const bool rv = row < valid;
        // ---- q . k for the G heads (16-byte slice per lane), summed over the row's lanes
        const uint4 ku = *reinterpret_cast<const uint4*>(sK + row * L::kRowBytes + lane_r * 16);
        const float2 k0 = bf16x2_to_f2(ku.x), k1 = bf16x2_to_f2(ku.y);
        const float2 k2 = bf16x2_to_f2(ku.z), k3 = bf16x2_to_f2(ku.w);
        float s[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 t = fmul2(qf[g][0], k0);
          t = ffma2(qf[g][1], k1, t);
          t = ffma2(qf[g][2], k2, t);
          t = ffma2(qf[g][3], k3, t);
          s[g] = t.x + t.y;
        }
        segment_allreduce<G, LPR>(s, seg_mask, lane_r);
        // ---- online softmax, per segment, with a stale max kept within 2^8
        bool need = false;
#pragma unroll
        for (int g = 0; g < G; ++g) need |= rv && (m[g] == -INFINITY || s[g] > m[g] + thr);
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            if (rv && (m[g] == -INFINITY || s[g] > m[g] + thr)) {
              const float alpha = (m[g] == -INFINITY) ? 0.f : ex2((m[g] - s[g]) * c2);
              l[g] *= alpha;
              const float2 al = make_float2(alpha, alpha);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[g][e] = fmul2(acc[g][e], al);
              m[g] = s[g];
            }
          }
        }
        if (rv) {
          const uint4 vu = *reinterpret_cast<const uint4*>(sV + row * L::kRowBytes + lane_r * 16);
          const float2 v0 = bf16x2_to_f2(vu.x), v1 = bf16x2_to_f2(vu.y);
          const float2 v2 = bf16x2_to_f2(vu.z), v3 = bf16x2_to_f2(vu.w);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pg = ex2(fmaf(s[g], c2, -m[g] * c2));
            l[g] += pg;
            const float2 p2 = make_float2(pg, pg);
            acc[g][0] = ffma2(p2, v0, acc[g][0]);
            acc[g][1] = ffma2(p2, v1, acc[g][1]);
            acc[g][2] = ffma2(p2, v2, acc[g][2]);
            acc[g][3] = ffma2(p2, v3, acc[g][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(EMPTY(stage));
    }
  }
  __syncthreads();   // ring no longer in use (the producer drained its copies)

  // ---- merge the per-segment states by log-sum-exp and write the split's partials
  float* ms = reinterpret_cast<float*>(smem);                 // [kStates][G] maxima
  float* ls = ms + L::kStates * G;                            // [kStates][G] sums
  float* os = ls + L::kStates * G;                            // [kStates][G][D] outputs
  if (warp < kConsumerWarps) {
    const int st = warp * SEGS + seg;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (lane_r == 0) {
        ms[st * G + g] = m[g];
        ls[st * G + g] = l[g];
      }
      float* dst = os + (static_cast<size_t>(st) * G + g) * D + lane_r * 8;
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
    }
  }
  __syncthreads();
  if (*abort_flag) return;
  const float c2 = a.scale_log2;
  const size_t row0 = (static_cast<size_t>(seq) * a.Hq + hkv * G) * a.max_splits + split;
  for (int idx = tid; idx < G * D; idx += kSplitThreads) {
    const int g = idx / D, col = idx % D;
    float M = -INFINITY;
    for (int e = 0; e < L::kStates; ++e) M = fmaxf(M, ms[e * G + g]);
    float tot = 0.f, o = 0.f;
    for (int e = 0; e < L::kStates; ++e) {
      const float me = ms[e * G + g];
      const float w = (me == -INFINITY) ? 0.f : ex2((me - M) * c2);
      tot = fmaf(w, ls[e * G + g], tot);
      o = fmaf(w, os[(static_cast<size_t>(e) * G + g) * D + col], o);
    }
    a.part_o[(row0 + static_cast<size_t>(g) * a.max_splits) * D + col] = o / tot;
    if (col == 0) a.part_lse[row0 + static_cast<size_t>(g) * a.max_splits] = fmaf(M, a.scale, __logf(tot));
  }
}

// ---------------------------------------------------------------------------
// Specialised split kernel for head dim 128 with 4 query heads per KV head
// (the common GQA shape).  Same work decomposition and results as
// decode_split_kernel, restructured to cut instructions per gathered byte:
//  * 8 warps, no dedicated producer: the last warp to finish a ring stage
//    (an acquire-release counter in shared memory) issues the stage's next
//    page copies, so every warp computes;
//  * each 16-lane row segment accumulates the partial q.k of its 4 rows of a
//    chunk before reducing: one reduce-scatter of 16 values leaves each lane
//    with exactly one (row, head) score, so each lane computes one
//    exponential per chunk and the stale-max check runs once per chunk;
//  * probabilities reach the P.V step through shared memory (one store, one
//    16-byte load per row) instead of shuffles;
//  * full chunks take a path without per-row validity checks.
// ---------------------------------------------------------------------------
constexpr int kG4Warps = 8;
constexpr int kG4Threads = 32 * kG4Warps;

struct G4Layout {
  static constexpr int D = 128;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunkBytes = kChunkTokens * kRowBytes;   // 16 KB
  static constexpr int kStageBytes = 2 * kChunkBytes;            // K then V
  static constexpr int kRing = kDecStages * kStageBytes;         // 96 KB
  static constexpr int kStates = kG4Warps * 2;                   // (warp, segment) softmax states
  static constexpr int kMerge = kStates * 4 * (D + 2) * 4;       // 33 KB, reuses the ring
  static constexpr int kProb = kRing;                            // [8 warps][2 seg][16] floats
  static constexpr int kTable = kProb + kG4Warps * 2 * 16 * 4;   // split's block-table entries
  static constexpr int kBar = kTable + kMaxSplitPages * 4;       // full[3]
  static constexpr int kCnt = kBar + kDecStages * 8;             // per-stage finish counters
  static constexpr int kMisc = kCnt + kDecStages * 4;            // abort flag, issued-chunk count
  static constexpr int kBytes = kMisc + 16;
  static_assert(kMerge <= kRing, "merge area fits in the ring");
};

__device__ __forceinline__ uint32_t atom_add_acq_rel_shared(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
  return old;
}

__global__ void __launch_bounds__(kG4Threads, 2) decode_split_g4_kernel(const DecodeArgs a) {
  using L = G4Layout;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem[];

  const int split = blockIdx.x, hkv = blockIdx.y, seq = blockIdx.z;
  const int raw_len = __ldg(a.seq_lens + seq);
  const int len = clamp_len(raw_len, a);
  if (raw_len != len && split == 0 && hkv == 0 && threadIdx.x == 0) atomicOr(a.status, kDevBadSeqLen);
  const int split_tokens = a.split_pages * a.page_size;
  const int t_begin = split * split_tokens;
  if (t_begin >= len) return;  // CTA-uniform: nothing in this split
  const int t_end = min(len, t_begin + split_tokens);
  const int n_chunks = (t_end - t_begin + kChunkTokens - 1) / kChunkTokens;
  const int split_first_page = split * a.split_pages;
  const int split_npages = (t_end - t_begin + a.page_size - 1) / a.page_size;
  const int pages_per_chunk = kChunkTokens / a.page_size;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = lane >> 4, lane_r = lane & 15;
  const uint32_t sbase = smem_u32(smem);
  int* tbl = reinterpret_cast<int*>(smem + L::kTable);
  float* sp = reinterpret_cast<float*>(smem + L::kProb) + (warp * 2 + seg) * 16;   // this segment's 16 weights
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);
  int* issued = reinterpret_cast<int*>(smem + L::kMisc + 4);   // chunks whose copies were issued
  auto FULL = [&](int s) { return sbase + L::kBar + 8u * s; };
  auto CNT = [&](int s) { return sbase + L::kCnt + 4u * s; };

  // index prefetch: the split's block-table entries, checked once
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(FULL(s), 1);
      reinterpret_cast<volatile uint32_t*>(smem + L::kCnt)[s] = 0;
    }
    *abort_flag = 0;
    *issued = min(kDecStages, n_chunks);
    fence_mbar_init();
  }
  load_split_table(a, seq, split_first_page, split_npages, tbl, tid, kG4Threads);
  __syncthreads();
  if (warp < kDecStages && warp < n_chunks) {
    const int first = warp * pages_per_chunk;
    const uint32_t st = sbase + warp * L::kStageBytes;
    gather_chunk<D>(a, hkv, tbl, first, min(pages_per_chunk, split_npages - first), st, st + L::kChunkBytes,
                    FULL(warp));
  }

  // q slices (16-byte slice lane_r of each of the 4 heads), fp32 pairs
  float2 qf[4][4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(a.q + (static_cast<size_t>(seq) * a.Hq + hkv * 4 + g) * D) +
                          lane_r);
    qf[g][0] = bf16x2_to_f2(u.x);
    qf[g][1] = bf16x2_to_f2(u.y);
    qf[g][2] = bf16x2_to_f2(u.z);
    qf[g][3] = bf16x2_to_f2(u.w);
  }
  // this lane's softmax state is that of head gh = lane_r & 3 of its segment;
  // acc holds the segment's partial output for all 4 heads on this d-slice
  const int gh = lane_r & 3, ph = lane_r >> 2;
  float m = -INFINITY, negmc = 0.f, l = 0.f;
  float2 acc[4][4];
#pragma unroll
  for (int g = 0; g < 4; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = make_float2(0.f, 0.f);
  const float c2 = a.scale_log2;
  const float thr = c2 > 0.f ? kDecRescaleLog2 / c2 : INFINITY;
  const uint32_t seg_mask = 0xFFFFu << (seg * 16);
  const int row_base = warp * 8 + seg;   // rows row_base + 2p, p = 0..3

  int c = 0;
  for (; c < n_chunks; ++c) {
    const int stage = c % kDecStages;
    const bool ok = mbar_wait(FULL(stage), (c / kDecStages) & 1u, a.status, abort_flag);
    if (!__all_sync(0xffffffffu, ok)) break;
    const int valid = min(kChunkTokens, t_end - (t_begin + c * kChunkTokens));
    const uint8_t* sK = smem + stage * L::kStageBytes + lane_r * 16;
    const uint8_t* sV = sK + L::kChunkBytes;
    if (warp * 8 < valid) {
      // ---- q . k of this segment's 4 rows, partial over this lane's 8 dims
      float v[16];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const uint4 ku = *reinterpret_cast<const uint4*>(sK + (row_base + 2 * p) * L::kRowBytes);
        const float2 k0 = bf16x2_to_f2(ku.x), k1 = bf16x2_to_f2(ku.y);
        const float2 k2 = bf16x2_to_f2(ku.z), k3 = bf16x2_to_f2(ku.w);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float2 t = fmul2(qf[g][0], k0);
          t = ffma2(qf[g][1], k1, t);
          t = ffma2(qf[g][2], k2, t);
          t = ffma2(qf[g][3], k3, t);
          v[p * 4 + g] = t.x + t.y;
        }
      }
      // ---- reduce-scatter the 16 (row, head) partials over the 16 lanes:
      // lane_r ends with the full score of (row p = lane_r >> 2, head lane_r & 3)
#pragma unroll
      for (int o = 8, n = 16; o >= 1; o >>= 1, n >>= 1) {
        const bool hi = lane_r & o;
#pragma unroll
        for (int k = 0; k < n / 2; ++k) {
          const float keep = hi ? v[k + n / 2] : v[k];
          const float send = hi ? v[k] : v[k + n / 2];
          v[k] = keep + __shfl_xor_sync(seg_mask, send, o);
        }
      }
      float sc = v[0];
      if (row_base + 2 * ph >= valid) sc = -INFINITY;
      // ---- online softmax for head gh over the chunk's 4 rows of this segment
      float cm = fmaxf(sc, __shfl_xor_sync(seg_mask, sc, 4));
      cm = fmaxf(cm, __shfl_xor_sync(seg_mask, cm, 8));
      const bool need = (cm != -INFINITY) && (m == -INFINITY || cm > m + thr);
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ((m == -INFINITY) ? 0.f : ex2((m - cm) * c2)) : 1.f;
        if (need) {
          m = cm;
          negmc = -cm * c2;
        }
        l *= alpha;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float ah = __shfl_sync(0xffffffffu, alpha, seg * 16 + h);
          const float2 a2 = make_float2(ah, ah);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][e] = fmul2(acc[h][e], a2);
        }
      }
      const float pv = (sc == -INFINITY) ? 0.f : ex2(fmaf(sc, c2, negmc));
      l += pv;
      sp[lane_r] = pv;
      __syncwarp();
      // ---- acc += p * v for the 4 rows
      if (valid == kChunkTokens) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float4 w4 = *reinterpret_cast<const float4*>(sp + 4 * p);
          const uint4 vu = *reinterpret_cast<const uint4*>(sV + (row_base + 2 * p) * L::kRowBytes);
          const float2 v0 = bf16x2_to_f2(vu.x), v1 = bf16x2_to_f2(vu.y);
          const float2 v2 = bf16x2_to_f2(vu.z), v3 = bf16x2_to_f2(vu.w);
          const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 w2 = make_float2(wv[h], wv[h]);
            acc[h][0] = ffma2(w2, v0, acc[h][0]);
            acc[h][1] = ffma2(w2, v1, acc[h][1]);
            acc[h][2] = ffma2(w2, v2, acc[h][2]);
            acc[h][3] = ffma2(w2, v3, acc[h][3]);
          }
        }
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (row_base + 2 * p < valid) {
            const float4 w4 = *reinterpret_cast<const float4*>(sp + 4 * p);
            const uint4 vu = *reinterpret_cast<const uint4*>(sV + (row_base + 2 * p) * L::kRowBytes);
            const float2 v0 = bf16x2_to_f2(vu.x), v1 = bf16x2_to_f2(vu.y);
            const float2 v2 = bf16x2_to_f2(vu.z), v3 = bf16x2_to_f2(vu.w);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float2 w2 = make_float2(wv[h], wv[h]);
              acc[h][0] = ffma2(w2, v0, acc[h][0]);
              acc[h][1] = ffma2(w2, v1, acc[h][1]);
              acc[h][2] = ffma2(w2, v2, acc[h][2]);
              acc[h][3] = ffma2(w2, v3, acc[h][3]);
            }
          }
        }
      }
      __syncwarp();
    }
    // ---- release the stage; the last warp to finish it issues its next copies
    uint32_t last = 0;
    if (lane == 0) last = (atom_add_acq_rel_shared(CNT(stage), 1u) == kG4Warps - 1) ? 1u : 0u;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      if (lane == 0) reinterpret_cast<volatile uint32_t*>(smem + L::kCnt)[stage] = 0;
      const int cn = c + kDecStages;
      if (cn < n_chunks) {
        fence_proxy_async_shared();   // generic reads of the stage before the async copies into it
        const int first = cn * pages_per_chunk;
        const uint32_t st = sbase + stage * L::kStageBytes;
        gather_chunk<D>(a, hkv, tbl, first, min(pages_per_chunk, split_npages - first), st, st + L::kChunkBytes,
                        FULL(stage));
        if (lane == 0) atomicMax(issued, cn + 1);
      }
    }
  }
  const bool aborted = c < n_chunks;
  __syncthreads();
  if (aborted || *abort_flag) {
    // a wait gave up: let whatever copies may be in flight land, then leave
    if (tid == 0) {
      const int hi = *reinterpret_cast<volatile int*>(issued);
      for (int cc = max(0, hi - kDecStages); cc < hi; ++cc)
        mbar_wait(FULL(cc % kDecStages), (cc / kDecStages) & 1u, nullptr, nullptr, kWaitLimitNs);
    }
    __syncthreads();
    return;
  }

  // ---- merge the 16 segment states by log-sum-exp, write the split's partials
  float* ms = reinterpret_cast<float*>(smem);
  float* ls = ms + L::kStates * 4;
  float* os = ls + L::kStates * 4;
  {
    const int st = warp * 2 + seg;
    float lt = l + __shfl_xor_sync(0xffffffffu, l, 4);
    lt += __shfl_xor_sync(0xffffffffu, lt, 8);
    if (ph == 0) {
      ms[st * 4 + gh] = m;
      ls[st * 4 + gh] = lt;
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float* dst = os + (static_cast<size_t>(st) * 4 + h) * D + lane_r * 8;
      reinterpret_cast<float4*>(dst)[0] = make_float4(acc[h][0].x, acc[h][0].y, acc[h][1].x, acc[h][1].y);
      reinterpret_cast<float4*>(dst)[1] = make_float4(acc[h][2].x, acc[h][2].y, acc[h][3].x, acc[h][3].y);
    }
  }
  __syncthreads();
  const size_t row0 = (static_cast<size_t>(seq) * a.Hq + hkv * 4) * a.max_splits + split;
  for (int idx = tid; idx < 4 * D; idx += kG4Threads) {
    const int g = idx / D, col = idx % D;
    float M = -INFINITY;
    for (int e = 0; e < L::kStates; ++e) M = fmaxf(M, ms[e * 4 + g]);
    float tot = 0.f, o = 0.f;
    for (int e = 0; e < L::kStates; ++e) {
      const float me = ms[e * 4 + g];
      const float w = (me == -INFINITY) ? 0.f : ex2((me - M) * c2);
      tot = fmaf(w, ls[e * 4 + g], tot);
      o = fmaf(w, os[(static_cast<size_t>(e) * 4 + g) * D + col], o);
    }
    a.part_o[(row0 + static_cast<size_t>(g) * a.max_splits) * D + col] = o / tot;
    if (col == 0) a.part_lse[row0 + static_cast<size_t>(g) * a.max_splits] = fmaf(M, a.scale, __logf(tot));
  }
}

template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeArgs a, __nv_bfloat16* o, float* lse) {
  const int hq = blockIdx.x, seq = blockIdx.y;
  const int len = clamp_len(__ldg(a.seq_lens + seq), a);
  const int split_tokens = a.split_pages * a.page_size;
  const int ns = (len + split_tokens - 1) / split_tokens;
  const size_t row0 = (static_cast<size_t>(seq) * a.Hq + hq) * a.max_splits;
  const size_t orow = static_cast<size_t>(seq) * a.Hq + hq;
  const int col = threadIdx.x;
  if (ns == 0) {
    if (col < D) o[orow * D + col] = __float2bfloat16(0.f);
    if (col == 0 && lse) lse[orow] = -INFINITY;
    return;
  }
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, a.part_lse[row0 + s]);
  float tot = 0.f, acc = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = __expf(a.part_lse[row0 + s] - mx);
    tot += w;
    if (col < D) acc = fmaf(w, a.part_o[(row0 + s) * D + col], acc);
  }
  if (col < D) o[orow * D + col] = __float2bfloat16(acc / tot);
  if (col == 0 && lse) lse[orow] = mx + __logf(tot);
}

// Gather-debug: the sequence's pages gathered split by split and chunk by
// chunk with the decode kernels' own table load and chunk copies, then written
// out contiguously.
template <int D>
__global__ void __launch_bounds__(kGatherThreads) gather_debug_kernel(const DecodeArgs a, int seq, int hkv,
                                                                   __nv_bfloat16* k_out, __nv_bfloat16* v_out) {
  using L = DecodeLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + L::kBar;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  int* tbl = reinterpret_cast<int*>(smem + L::kTable);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int raw_len = __ldg(a.seq_lens + seq);
  const int len = clamp_len(raw_len, a);
  if (tid == 0) {
    if (raw_len != len) atomicOr(a.status, kDevBadSeqLen);
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int pages_per_chunk = kChunkTokens / a.page_size;
  const int split_tokens = a.split_pages * a.page_size;
  int phase = 0;
  for (int t_begin = 0, split = 0; t_begin < len; t_begin += split_tokens, ++split) {
    const int t_end = min(len, t_begin + split_tokens);
    const int split_npages = (t_end - t_begin + a.page_size - 1) / a.page_size;
    load_split_table(a, seq, split * a.split_pages, split_npages, tbl, tid, kGatherThreads);
    __syncthreads();
    for (int first = 0; first < split_npages; first += pages_per_chunk) {
      const int npg = min(pages_per_chunk, split_npages - first);
      if (warp == 0) {
        fence_proxy_async_shared();   // earlier generic reads of the staging area before the async copies
        gather_chunk<D>(a, hkv, tbl, first, npg, sbase, sbase + L::kChunkBytes, bar);
      }
      const bool ok = mbar_wait(bar, phase & 1u, a.status, abort_flag);
      phase++;
      if (__syncthreads_or(!ok)) {
        // a wait gave up: let the copies in flight land before leaving
        if (tid == 0) mbar_wait(bar, (phase - 1) & 1u, nullptr, nullptr, kWaitLimitNs);
        __syncthreads();
        return;
      }
      const int t0 = t_begin + first * a.page_size;
      const int rows = min(npg * a.page_size, len - t0);
      const int words = rows * D / 8;   // 16-byte words
      for (int w = tid; w < words; w += kGatherThreads) {
        reinterpret_cast<uint4*>(k_out + static_cast<size_t>(t0) * D)[w] = reinterpret_cast<const uint4*>(smem)[w];
        reinterpret_cast<uint4*>(v_out + static_cast<size_t>(t0) * D)[w] =
            reinterpret_cast<const uint4*>(smem + L::kChunkBytes)[w];
      }
      __syncthreads();
    }
  }
}

// Bounded-wait self-test: nothing ever arrives on this barrier.
__global__ void selftest_wait_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  fence_mbar_init();
  mbar_wait(b, 0, status, &abort_flag, limit_ns);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static DecodeArgs make_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                            const int32_t* seq_lens, int page_size, int num_seqs, int Hq, int Hkv, int max_pages,
                            int num_pages_total, float scale, int split_pages, int max_splits, void* workspace,
                            const DecodePlan* plan, unsigned* status) {
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_cache = static_cast<const uint8_t*>(k_cache);
  a.v_cache = static_cast<const uint8_t*>(v_cache);
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.page_size = page_size;
  a.num_seqs = num_seqs;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.max_pages = max_pages;
  a.num_pages_total = num_pages_total;
  a.split_pages = split_pages;
  a.max_splits = max_splits;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.part_o = plan ? reinterpret_cast<float*>(ws + plan->partial_o_offset) : nullptr;
  a.part_lse = plan ? reinterpret_cast<float*>(ws + plan->partial_lse_offset) : nullptr;
  a.status = status;
  return a;
}

template <int D, int G>
static cudaError_t launch_split(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  using L = DecodeLayout<D>;
  static int attr_done[64] = {0};
  cudaError_t e = ensure_smem_limit(decode_split_kernel<D, G>, L::kBytes, attr_done);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D, G><<<grid, kSplitThreads, L::kBytes, stream>>>(a);
  return cudaGetLastError();
}

static cudaError_t launch_split_g4(const DecodeArgs& a, dim3 grid, cudaStream_t stream) {
  static int attr_done[64] = {0};
  cudaError_t e = ensure_smem_limit(decode_split_g4_kernel, G4Layout::kBytes, attr_done);
  if (e != cudaSuccess) return e;
  decode_split_g4_kernel<<<grid, kG4Threads, G4Layout::kBytes, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_split_g(const DecodeArgs& a, int G, dim3 grid, cudaStream_t stream) {
  if (D == 128 && G == 4) return launch_split_g4(a, grid, stream);
  switch (G) {
    case 1: return launch_split<D, 1>(a, grid, stream);
    case 2: return launch_split<D, 2>(a, grid, stream);
    case 4: return launch_split<D, 4>(a, grid, stream);
    default: return launch_split<D, 8>(a, grid, stream);
  }
}

ta_status launch_paged_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                              const int32_t* seq_lens, int page_size, int num_seqs, int Hq, int Hkv, int d,
                              int max_pages, int num_pages_total, float scale, void* o, float* lse, void* workspace,
                              const DecodePlan& plan, cudaStream_t stream) {
  if (num_seqs == 0) return TA_OK;
  unsigned* status = static_cast<unsigned*>(workspace);
  cudaError_t me = cudaMemsetAsync(status, 0, sizeof(unsigned), stream);
  if (me != cudaSuccess) return fail(TA_ERR_CUDA, "decode: status reset", me);
  DecodeArgs a = make_args(q, k_cache, v_cache, block_table, seq_lens, page_size, num_seqs, Hq, Hkv, max_pages,
                           num_pages_total, scale, plan.split_pages, plan.max_splits, workspace, &plan, status);
  const int G = Hq / Hkv;
  dim3 grid(plan.max_splits, Hkv, num_seqs);
  cudaError_t e = (d == 128) ? launch_split_g<128>(a, G, grid, stream) : launch_split_g<64>(a, G, grid, stream);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "decode: split kernel launch", e);
  dim3 cgrid(Hq, num_seqs);
  if (d == 128)
    decode_combine_kernel<128><<<cgrid, 128, 0, stream>>>(a, static_cast<__nv_bfloat16*>(o), lse);
  else
    decode_combine_kernel<64><<<cgrid, 128, 0, stream>>>(a, static_cast<__nv_bfloat16*>(o), lse);
  e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "decode: combine kernel launch", e);
}

ta_status launch_gather_debug(const void* k_cache, const void* v_cache, const int32_t* block_table,
                              const int32_t* seq_lens, int seq, int hkv, int page_size, int Hkv, int d,
                              int max_pages, int num_pages_total, void* k_out, void* v_out, cudaStream_t stream) {
  unsigned* status = device_status_ptr();
  if (!status) return TA_ERR_CUDA;
  // splits as the decode plan forms them for a batch that fills the GPU
  const int split_pages = (kSplitTokens / page_size < kMaxSplitPages) ? kSplitTokens / page_size : kMaxSplitPages;
  DecodeArgs a = make_args(nullptr, k_cache, v_cache, block_table, seq_lens, page_size, seq + 1, Hkv, Hkv, max_pages,
                           num_pages_total, 1.f, split_pages, 1, nullptr, nullptr, status);
  static int done128[64] = {0}, done64[64] = {0};
  if (d == 128) {
    if (ensure_smem_limit(gather_debug_kernel<128>, DecodeLayout<128>::kBytes, done128) != cudaSuccess)
      return TA_ERR_CUDA;
    gather_debug_kernel<128><<<1, kGatherThreads, DecodeLayout<128>::kBytes, stream>>>(
        a, seq, hkv, static_cast<__nv_bfloat16*>(k_out), static_cast<__nv_bfloat16*>(v_out));
  } else {
    if (ensure_smem_limit(gather_debug_kernel<64>, DecodeLayout<64>::kBytes, done64) != cudaSuccess)
      return TA_ERR_CUDA;
    gather_debug_kernel<64><<<1, kGatherThreads, DecodeLayout<64>::kBytes, stream>>>(
        a, seq, hkv, static_cast<__nv_bfloat16*>(k_out), static_cast<__nv_bfloat16*>(v_out));
  }
  return cudaGetLastError() == cudaSuccess ? TA_OK : TA_ERR_CUDA;
}

ta_status launch_selftest_wait(unsigned limit_us, cudaStream_t stream) {
  unsigned* status = device_status_ptr();
  if (!status) return TA_ERR_CUDA;
  selftest_wait_kernel<<<1, 1, 0, stream>>>(status, static_cast<unsigned long long>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? TA_OK : TA_ERR_CUDA;
}

// SMs of the current device; 148 (B200) when no device can be queried, so a
// size query made without a GPU still gets the plan a B200 would use.
static int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();   // clear the non-sticky error of the failed query
    return 148;
  }
  return n;
}

bool make_decode_plan(int num_seqs, int Hq, int Hkv, int d, int max_pages, int page_size, DecodePlan* plan) {
  if (page_size != 8 && page_size != 16 && page_size != 32 && page_size != 64) return false;
  if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || max_pages <= 0 || (d != 64 && d != 128)) return false;
  const int chunk_pages = kChunkTokens / page_size;
  int sp = kSplitTokens / page_size;
  if (sp > kMaxSplitPages) sp = kMaxSplitPages;   // the split's table holds kMaxSplitPages entries
  // enough CTAs to balance uneven lengths: 8 per SM of the current device
  const long long target = 8LL * current_sm_count();
  auto splits_for = [&](int p) { return (max_pages + p - 1) / p; };
  while (sp > chunk_pages && static_cast<long long>(num_seqs) * Hkv * splits_for(sp) < target) sp /= 2;
  if (sp < chunk_pages) sp = chunk_pages;
  plan->chunk_tokens = kChunkTokens;
  plan->split_pages = sp;
  plan->max_splits = splits_for(sp);
  const size_t rows = static_cast<size_t>(num_seqs) * Hq * plan->max_splits;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  plan->partial_o_offset = 256;
  plan->partial_lse_offset = up(plan->partial_o_offset + rows * d * sizeof(float));
  plan->bytes = up(plan->partial_lse_offset + rows * sizeof(float));
  return true;
}

}  // namespace ta
