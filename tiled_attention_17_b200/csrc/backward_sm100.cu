// Attention backward for sm_100a (B200): gradients dQ, dK, dV of
// O = softmax(scale * Q K^T [+ causal mask]) V, by recomputation.
//
// The forward pass keeps only each row's log-sum-exp; the backward pass
// recomputes the Q K^T blocks from it and streams the gradients tile by tile,
// so neither S nor P is ever stored (Gemini 3 Flash kernel-fusion post,
// section 4, recomputation strategy).  With P = exp(S - lse) per row:
//
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - delta),  delta_i = dO_i . O_i
//   dQ = scale dS K,  dK = scale dS^T Q
//
// (delta_i equals sum_j P_ij dP_ij, the softmax Jacobian's row term, because
// O_i = sum_j P_ij v_j.)  Three kernels:
//   bwd_prep_kernel    delta and lse (in log2 units, +inf for rows with no
//                      visible key) per query row, into a padded workspace
//   bwd_dkdv_kernel    one CTA per 128-key tile of one (batch, KV head); loops
//                      over the query heads of the group and the query tiles
//                      that see the keys; dK, dV accumulate in TMEM
//   bwd_dq_kernel      one CTA per 128-row query tile; loops over key tiles;
//                      dQ accumulates in TMEM
// Splitting dQ from dK/dV recomputes S and dP once more (7 tile GEMMs instead
// of 5) but needs no atomics, so the gradients are deterministic.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// tcgen05.mma issuer (the whole warp runs the loop, one elected lane
// issues), warps 4-11 two warpgroups for the elementwise work and the
// epilogue: thread (h, row) owns one tile row's
// columns [64h, 64h + 64).  The elementwise steps need no row reduction (the
// row statistics come precomputed), so the two halves never exchange data;
// each writes its bf16 result over the TMEM columns it read, and the
// accumulating products take the two halves as separate A addresses.  All operand forms are the forward
// kernel's: K-major A and B from shared memory for the score-like products,
// bf16 probabilities from TMEM as A with an MN-major B for the accumulating
// ones.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "ptx.cuh"
#include "tiledattn_internal.h"

namespace ta {
namespace {

constexpr int kT = 128;          // rows per tile (queries or keys)
constexpr int kBwdThreads = 384;
constexpr int kWorkWarp0 = 4;    // warps 4-11: thread (h, row) owns columns [64h, 64h + 64) of a tile row
// Launch at 168 registers per thread (one warp of each of the three
// warpgroups per sub-partition: 3 x 168 = 504 of 512), then re-split.
constexpr int kBwdLaunchRegs = 168;
constexpr int kBwdRegsControl = 120;
constexpr int kBwdRegsWork = 192;
static_assert(kBwdRegsControl + 2 * kBwdRegsWork <= 3 * kBwdLaunchRegs, "register split");

template <int D>
struct BwdTiles {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kChunks = D / 64;              // 64-column (128-byte) swizzle atoms
  static constexpr int kTileBytes = kT * D * 2;
  static constexpr int kChunkBytes = kT * 128;
};

struct BwdArgs {
  int B, Hq, Hkv, Nq, Nkv;
  int n_qt, n_kt;              // query / key tiles per head
  int causal;
  float scale;                 // multiplies dQ and dK
  float scale_log2;            // scale * log2(e)
  const float* delta;          // [B*Hq][n_qt*128]
  const float* lse2;           // [B*Hq][n_qt*128], log2 units, +inf = no visible key
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  unsigned* status;
  // Items are launched in groups of heads (dK/dV: KV heads, dQ: query heads),
  // all of a group's tiles before the next group's, heaviest tile first
  // within the group.  The CTAs running at once then stream one or two
  // groups' operands instead of every head's, so each streamed tile is read
  // from DRAM about once.  The host sizes the groups (L2 and load-balance
  // bounds, launch_bwd_d); one group is the tile-major order across all heads.
  int kv_group, q_group;
};

// The elected lane issues a whole product inside one branch: a branch per
// MMA (the warp splitting and reconverging around every instruction) made
// issue, at ~50 cycles per MMA, as slow as the tensor pipe executes a
// 128 x 128 x 16 step, so the pipe sat idle between instructions.

// D = A B^T with A, B K-major operand tiles (128 rows x D, 128-byte swizzle):
// descriptor of the tile, +2 per 16-element step inside a 64-column chunk,
// +chunk to the next.
template <int kChunks>
__device__ __forceinline__ void mma_kmajor_tile(bool leader, uint32_t d_tmem, uint64_t a0, uint64_t b0,
                                                uint32_t idesc) {
  if (leader) {
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4)
        mma_ss(d_tmem, a0 + c * ((kT * 128) >> 4) + 2 * k4, b0 + c * ((kT * 128) >> 4) + 2 * k4, idesc,
               (c | k4) != 0 ? 1u : 0u);
  }
  __syncwarp();
}

// D += A B with A = 128 x 128 bf16 in TMEM (packed pairs: K = 0..63 in the 32
// columns at a_lo, K = 64..127 in the 32 columns at a_hi) and B = an MN-major
// 128-row x D tile in shared memory (K = its rows).
__device__ __forceinline__ void mma_tmem_a(bool leader, uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint64_t b0,
                                           uint32_t idesc, bool acc) {
  if (leader) {
    const uint32_t acc0 = acc ? 1u : 0u;
#pragma unroll
    for (int kk = 0; kk < kT / 16; ++kk)
      mma_ts(d_tmem, (kk < 4 ? a_lo : a_hi - 32) + kk * 8, b0 + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc,
             kk > 0 ? 1u : acc0);
  }
  __syncwarp();
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// P^T over 64 query columns of one key row: p_c = exp2(s_c c2 - lse2_c) as
// bf16 pairs.  The caller loads the columns' lse2 into registers (lv) before
// it waits for S^T, so those shared-memory loads, which queue behind the
// tensor pipe's operand reads, overlap the wait instead of the
// exponentials.  kMask zeroes the columns c < lo (causally hidden, or every
// column of a key row past the keys).  The two forms are separate code
// paths behind a warp-uniform branch: a compare-and-select per element on
// every tile would cost more issue slots than the exponentials themselves.
template <bool kMask>
__device__ __forceinline__ void p_row_half(const float* sv, const float4* lv, float c2, int lo, uint32_t* pk) {
#pragma unroll
  for (int e4 = 0; e4 < 16; ++e4) {
    const float4 l4 = lv[e4];
    const int c = 4 * e4;
    float p0 = ex2(fmaf(sv[c + 0], c2, -l4.x)), p1 = ex2(fmaf(sv[c + 1], c2, -l4.y));
    float p2 = ex2(fmaf(sv[c + 2], c2, -l4.z)), p3 = ex2(fmaf(sv[c + 3], c2, -l4.w));
    if constexpr (kMask) {
      p0 = c + 0 >= lo ? p0 : 0.f;
      p1 = c + 1 >= lo ? p1 : 0.f;
      p2 = c + 2 >= lo ? p2 : 0.f;
      p3 = c + 3 >= lo ? p3 : 0.f;
    }
    pk[2 * e4] = pack_bf16x2(p0, p1);
    pk[2 * e4 + 1] = pack_bf16x2(p2, p3);
  }
}

// dS over 64 key columns of one query row: P = exp2(s_c c2 - lse2), rounded
// to bf16 as the dK/dV kernel rounds it, times (dP_c - delta).  kMask zeroes
// the columns c >= lim (causally hidden or past the keys).
template <bool kMask>
__device__ __forceinline__ void ds_row_half(const float* sv, const float* dpv, float c2, float l2, float dl, int lim,
                                            uint32_t* pk) {
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int c = 2 * e;
    float p0 = ex2(fmaf(sv[2 * e], c2, -l2));
    float p1 = ex2(fmaf(sv[2 * e + 1], c2, -l2));
    if constexpr (kMask) {
      p0 = c < lim ? p0 : 0.f;
      p1 = c + 1 < lim ? p1 : 0.f;
    }
    const uint32_t pb = pack_bf16x2(p0, p1);
    pk[e] = pack_bf16x2(bf16lo(pb) * (dpv[2 * e] - dl), bf16hi(pb) * (dpv[2 * e + 1] - dl));
  }
}

// ---------------------------------------------------------------------------
// delta_i = dO_i . O_i and lse in log2 units per (padded) query row
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ delta,
                                                       float* __restrict__ lse2, int Nq, int n_rows_pad,
                                                       long long total_pad) {
  // 8 lanes per row, each covering D/8 contiguous elements
  constexpr int kPer = D / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long r = gt >> 3;
  const int part = static_cast<int>(gt & 7);
  if (r >= total_pad) return;   // whole 8-lane groups leave together
  const long long bh = r / n_rows_pad;
  const int i = static_cast<int>(r - bh * n_rows_pad);
  float acc = 0.f;
  if (i < Nq) {
    const size_t off = (static_cast<size_t>(bh) * Nq + i) * D + part * kPer;
    const uint4* po = reinterpret_cast<const uint4*>(o + off);
    const uint4* pd = reinterpret_cast<const uint4*>(dout + off);
#pragma unroll
    for (int v = 0; v < kPer / 8; ++v) {
      const uint4 a = po[v], b = pd[v];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) acc += bf16lo(aw[e]) * bf16lo(bw[e]) + bf16hi(aw[e]) * bf16hi(bw[e]);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (part == 0) {
    delta[r] = acc;
    float l2 = INFINITY;
    if (i < Nq) {
      const float l = lse[static_cast<size_t>(bh) * Nq + i];
      if (l != -INFINITY) l2 = l * 1.4426950408889634f;
    }
    lse2[r] = l2;
  }
}

// ---------------------------------------------------------------------------
// dK, dV: work items are (key tile, batch, KV head), key tiles that more
// query tiles see first.  As in the dQ kernel, a CTA runs its own item and
// then takes over the items of CTAs not yet launched (cluster launch
// control).  The Q/dO ring and the S, P, dP and dS hand-offs run on across
// items as one stream of (query head, query tile) pairs: the next key tile's
// K and V load as soon as the current tile's last S^T and dP^T are issued,
// and its first S^T and dP^T follow the current tile's last dV and dK while
// the work warps write dK and dV out.
// ---------------------------------------------------------------------------
template <int D>
struct DkdvLayout {
  using T = BwdTiles<D>;
  static constexpr int kK = 0;
  static constexpr int kV = kK + T::kTileBytes;
  static constexpr int kQ = kV + T::kTileBytes;              // 2 stages
  static constexpr int kDO = kQ + 2 * T::kTileBytes;         // 2 stages
  static constexpr int kVec = kDO + 2 * T::kTileBytes;       // 2 stages x {lse2, delta} x 128 floats
  static constexpr int kBar = kVec + 2 * 2 * kT * 4;
  // kv_full, kv_empty, q_full[2], q_empty[2], s_full, p_full, dp_full, ds_full, acc_done, acc_empty,
  // item_full[2], item_empty[2], fin
  static constexpr int kNumBars = 17;
  static constexpr int kResp = (kBar + kNumBars * 8 + 15) & ~15;   // two 16-byte work-request answers
  static constexpr int kMisc = kResp + 32;
  static constexpr int kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "dynamic shared memory per block");
  // TMEM: S^T | dP^T | dV | dK
  static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDV = 256, kTmDK = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
};

// First query tile whose rows see key tile kt (bottom-right causal alignment:
// query q sees key k iff k <= q + Nkv - Nq).
__host__ __device__ inline int first_query_tile(int kt, const BwdArgs& a) {
  if (!a.causal) return 0;
  const int q_min = kt * kT - (a.Nkv - a.Nq);   // smallest query that sees the tile's first key
  return q_min <= 0 ? 0 : q_min / kT;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdArgs a) {
  using T = BwdTiles<D>;
  using L = DkdvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sK = sb + L::kK, sV = sb + L::kV, sQ = sb + L::kQ, sDO = sb + L::kDO;
  const float* vec = reinterpret_cast<const float*>(smem + L::kVec);
  const uint32_t bar0 = sb + L::kBar;
  // kv_empty: the key tile's last S^T and dP^T have read K and V; acc_empty:
  // the epilogue has read dV and dK; item_full / item_empty: a work request's
  // answer has landed / has been read by every consumer
  const uint32_t BAR_KV = bar0, BAR_KVE = bar0 + 8u;
  auto BAR_QF = [&](int s) { return bar0 + 8u * (2 + s); };
  auto BAR_QE = [&](int s) { return bar0 + 8u * (4 + s); };
  const uint32_t BAR_SF = bar0 + 8u * 6, BAR_PF = bar0 + 8u * 7, BAR_DPF = bar0 + 8u * 8,
                 BAR_DSF = bar0 + 8u * 9, BAR_ACC = bar0 + 8u * 10, BAR_ACCE = bar0 + 8u * 11,
                 BAR_FIN = bar0 + 8u * 16;
  auto BAR_ITF = [&](int s) { return bar0 + 8u * (12 + s); };
  auto BAR_ITE = [&](int s) { return bar0 + 8u * (14 + s); };
  const uint32_t sResp = sb + L::kResp;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the dQ kernel, launched as a programmatic dependent, may start as SMs free up
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int bh_count = a.B * a.Hkv;
  const int G = a.Hq / a.Hkv;
  struct Item {
    int kt, b, hkv, i0, per_head, n;   // n: (query head of the group, query tile) pairs
  };
  auto decode_item = [&](int idx) {
    Item it;
    const int grp = idx / (a.kv_group * a.n_kt), base = grp * a.kv_group;
    const int in_grp = min(a.kv_group, bh_count - base), rem = idx - grp * a.kv_group * a.n_kt;
    it.kt = rem / in_grp;
    const int bhk = base + rem % in_grp;
    it.b = bhk / a.Hkv;
    it.hkv = bhk % a.Hkv;
    it.i0 = first_query_tile(it.kt, a);
    it.per_head = it.i0 < a.n_qt ? a.n_qt - it.i0 : 0;
    it.n = G * it.per_head;
    return it;
  };
  // Work request k >= 1 (the item after the k-th) answers in slot k & 1; it is
  // that slot's ((k - 1) >> 1)-th use.
  auto resp_parity = [](int k) { return static_cast<uint32_t>((k - 1) >> 1) & 1u; };

  if (threadIdx.x == 0) {
    mbar_init(BAR_KV, 1);
    mbar_init(BAR_KVE, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR_QF(s), 1);
      mbar_init(BAR_QE(s), 1);
      mbar_init(BAR_ITF(s), 1);
      mbar_init(BAR_ITE(s), 1 + 256);   // the MMA warp's leader and every work thread
    }
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_PF, 256);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_DSF, 256);
    mbar_init(BAR_ACC, 1);
    mbar_init(BAR_ACCE, 256);
    mbar_init(BAR_FIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < kWorkWarp0) {
  setmaxnreg_dec<kBwdRegsControl>();
  if (warp == 0 && lane == 0) {
    // ======================= TMA producer =======================
    bool ok = true;
    uint32_t u = 0;   // (query head, query tile) pairs loaded so far: ring stage u & 1, use u >> 1
    int qi = 0;       // key tiles whose K and V were loaded
    int requested = 0, answered = 0;
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0 && ok; ++k) {
      // ask for the item after this one now, so the answer is back when it is needed
      {
        const int kn = k + 1, sl = kn & 1;
        if (kn >= 3 && !(ok = mbar_wait(BAR_ITE(sl), resp_parity(kn - 2), a.status, abort_flag))) break;
        fence_proxy_async_smem();   // the slot's previous answer was read through the generic proxy
        mbar_arrive_expect_tx(BAR_ITF(sl), 16);
        clc_try_cancel(sResp + 16 * sl, BAR_ITF(sl));
        requested = kn;
      }
      const Item it = decode_item(idx);
      if (it.n > 0) {
        // K and V are free once the previous key tile's last S^T and dP^T completed
        if (qi > 0 && !(ok = mbar_wait(BAR_KVE, static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag))) break;
        const int zk = it.b * a.Hkv + it.hkv;
        mbar_arrive_expect_tx(BAR_KV, 2 * T::kTileBytes);
        tma_load_4d(sK, &tmK, BAR_KV, 0, it.kt * kT, 0, zk);
        tma_load_4d(sV, &tmV, BAR_KV, 0, it.kt * kT, 0, zk);
        ++qi;
        for (int j = 0; j < it.n; ++j) {
          const int s = static_cast<int>(u & 1u);
          if (!(ok = mbar_wait(BAR_QE(s), ((u >> 1) & 1u) ^ 1u, a.status, abort_flag))) break;
          const int hq = it.hkv * G + j / it.per_head, qt = it.i0 + j % it.per_head;
          const int zq = it.b * a.Hq + hq;
          mbar_arrive_expect_tx(BAR_QF(s), 2 * T::kTileBytes + 2 * kT * 4);
          tma_load_4d(sQ + s * T::kTileBytes, &tmQ, BAR_QF(s), 0, qt * kT, 0, zq);
          tma_load_4d(sDO + s * T::kTileBytes, &tmDO, BAR_QF(s), 0, qt * kT, 0, zq);
          const size_t vrow = static_cast<size_t>(zq) * (a.n_qt * kT) + qt * kT;
          bulk_load(sb + L::kVec + (s * 2 + 0) * kT * 4, a.lse2 + vrow, kT * 4, BAR_QF(s));
          bulk_load(sb + L::kVec + (s * 2 + 1) * kT * 4, a.delta + vrow, kT * 4, BAR_QF(s));
          ++u;
        }
        if (!ok) break;
      }
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
      answered = kn;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
    }
    // drain: no copy into this CTA's shared memory may still be in flight at exit
    if (answered < requested)
      mbar_wait(BAR_ITF(requested & 1), resp_parity(requested), nullptr, nullptr, kWaitLimitNs);
    if (qi > 0) mbar_wait(BAR_KV, static_cast<uint32_t>(qi - 1) & 1u, nullptr, nullptr, kWaitLimitNs);
    for (uint32_t g = (u > 2u ? u - 2u : 0u); g < u; ++g)
      mbar_wait(BAR_QF(static_cast<int>(g & 1u)), (g >> 1) & 1u, nullptr, nullptr, kWaitLimitNs);
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    // The whole warp runs the issue loop (warp-uniform descriptors and
    // waits); the elected lane issues the MMAs and their commits.
    const bool leader = elect_one_sync();
    auto commit = [&](uint32_t bar) {
      if (leader) mma_commit(bar);
      __syncwarp();
    };
    constexpr uint32_t idesc_s = idesc_bf16_f32(kT, kT, false);   // 128 x 128, K-major B
    constexpr uint32_t idesc_acc = idesc_bf16_f32(kT, D, true);   // 128 x D, MN-major B
    const uint64_t dK = smem_desc_sw128(sK, 16, 1024), dV = smem_desc_sw128(sV, 16, 1024);
    const uint64_t dQk = smem_desc_sw128(sQ, 16, 1024), dDOk = smem_desc_sw128(sDO, 16, 1024);
    const uint64_t dQm = smem_desc_sw128(sQ, T::kChunkBytes, 1024), dDOm = smem_desc_sw128(sDO, T::kChunkBytes, 1024);
    constexpr uint64_t kStep = T::kTileBytes >> 4;
    bool ok = true;
    uint32_t u = 0;   // (query head, query tile) pairs so far: ring stage and hand-off phases
    int qi = 0;       // key tiles with work so far
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0 && ok; ++k) {
      const Item it = decode_item(idx);
      if (it.n > 0) {
        // the first pair's S^T = K Q^T and dP^T = V dO^T: this key tile's K and V
        // and the pair's Q stage have landed; the previous tile's last dV and dK
        // were issued before these, so they read P^T and dS^T first
        if (!(ok = mbar_wait_warp(BAR_KV, static_cast<uint32_t>(qi) & 1u, a.status, abort_flag))) break;
        if (!(ok = mbar_wait_warp(BAR_QF(static_cast<int>(u & 1u)), (u >> 1) & 1u, a.status, abort_flag))) break;
        tc_fence_after();
        mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmS, dK, dQk + (u & 1u) * kStep, idesc_s);
        commit(BAR_SF);
        mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmDP, dV, dDOk + (u & 1u) * kStep, idesc_s);
        commit(BAR_DPF);
        if (it.n == 1) commit(BAR_KVE);
        for (int j = 0; j < it.n; ++j) {
          const uint32_t uj = u + static_cast<uint32_t>(j);
          const int s = static_cast<int>(uj & 1u), s1 = s ^ 1;
          const uint32_t ph = uj & 1u;
          // dV += P^T dO once P^T is in TMEM; a key tile's first product
          // overwrites the accumulators, which the previous epilogue must have read
          if (!(ok = mbar_wait_warp(BAR_PF, ph, a.status, abort_flag))) break;
          if (j == 0 && qi > 0 &&
              !(ok = mbar_wait_warp(BAR_ACCE, static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag)))
            break;
          tc_fence_after();
          mma_tmem_a(leader, tmem + L::kTmDV, tmem + L::kTmS, tmem + L::kTmS + 64, dDOm + s * kStep, idesc_acc, j > 0);
          // next pair's S^T: the S buffer is free once the dV product above has read P^T
          if (j + 1 < it.n) {
            if (!(ok = mbar_wait_warp(BAR_QF(s1), ((uj + 1) >> 1) & 1u, a.status, abort_flag))) break;
            tc_fence_after();
            mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmS, dK, dQk + s1 * kStep, idesc_s);
            commit(BAR_SF);
          }
          // dK += dS^T Q once dS^T is in TMEM
          if (!(ok = mbar_wait_warp(BAR_DSF, ph, a.status, abort_flag))) break;
          tc_fence_after();
          mma_tmem_a(leader, tmem + L::kTmDK, tmem + L::kTmDP, tmem + L::kTmDP + 64, dQm + s * kStep, idesc_acc, j > 0);
          commit(BAR_QE(s));   // this stage's Q, dO, lse and delta are read once these land
          if (j + 1 < it.n) {
            mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmDP, dV, dDOk + s1 * kStep, idesc_s);
            commit(BAR_DPF);
            if (j + 2 == it.n) commit(BAR_KVE);   // the key tile's last S^T and dP^T: K and V are free
          }
        }
        if (!ok) break;
        commit(BAR_ACC);
        u += static_cast<uint32_t>(it.n);
        ++qi;
      }
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = mbar_wait_warp(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      __syncwarp();
      if (leader) mbar_arrive(BAR_ITE(sl));
    }
    // no commit may still be pending when the CTA exits
    commit(BAR_FIN);
    mbar_wait_warp(BAR_FIN, 0, nullptr, nullptr);
  }
  } else {
    setmaxnreg_inc<kBwdRegsWork>();
    // ======================= per-key-row work + epilogue =======================
    const int h = (warp - kWorkWarp0) / 4;         // query columns [64h, 64h + 64) of each tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c2 = a.scale_log2;
    const int off = a.Nkv - a.Nq;
    bool ok = true;
    uint32_t u = 0;   // (query head, query tile) pairs so far
    int qi = 0;       // key tiles with work so far
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0; ++k) {
      const Item it = decode_item(idx);
      const int key = it.kt * kT + r;
      for (int j = 0; j < it.n && ok; ++j) {
        const uint32_t uj = u + static_cast<uint32_t>(j);
        const int s = static_cast<int>(uj & 1u);
        const uint32_t ph = uj & 1u;
        const int qt = it.i0 + j % it.per_head;
        const int q0 = qt * kT;
        // query columns c with key > q0 + c + off are masked: c < lim
        const int lim = (a.causal ? key - off - q0 : 0) - h * 64;
        const bool row_ok = key < a.Nkv;
        const bool need_mask = !row_ok || lim > 0;
        ok = mbar_wait(BAR_QF(s), (uj >> 1) & 1u, a.status, abort_flag);
        const float* l2v = vec + (s * 2 + 0) * kT + h * 64;
        const float* dlv = vec + (s * 2 + 1) * kT + h * 64;
        // this half's 64 lse2 values into registers while S^T is computed
        float4 lv[16];
#pragma unroll
        for (int e4 = 0; e4 < 16; ++e4) lv[e4] = reinterpret_cast<const float4*>(l2v)[e4];
        ok = ok && mbar_wait(BAR_SF, ph, a.status, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // P^T = exp2(S^T c2 - lse2[query]) over this half's 64 query columns,
        // written as bf16 over the first 32 of the columns it was read from
        uint32_t pk[32];
        {
          uint32_t sr[2][32];
          tmem_ld32(tmem + L::kTmS + lane_off + h * 64, sr[0]);
          tmem_ld32(tmem + L::kTmS + lane_off + h * 64 + 32, sr[1]);
          tmem_wait_ld();
          const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
          // lanes that need no mask have lim <= 0 and keep every column
          if (__any_sync(0xffffffffu, need_mask))
            p_row_half<true>(sv, lv, c2, row_ok ? lim : 64, pk);
          else
            p_row_half<false>(sv, lv, c2, 0, pk);
          tmem_st32(tmem + L::kTmS + lane_off + h * 64, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR_PF);
        // dS^T = P^T o (dP^T - delta[query]) over this half, written over dP^T; delta
        // into registers while dP^T is computed
        float4 dv4[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) dv4[e2] = reinterpret_cast<const float4*>(dlv)[e2];
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR_DPF, ph, a.status, abort_flag)))) break;
        tc_fence_after();
        {
          uint32_t dr[2][32];
          tmem_ld32(tmem + L::kTmDP + lane_off + h * 64, dr[0]);
          tmem_ld32(tmem + L::kTmDP + lane_off + h * 64 + 32, dr[1]);
          tmem_wait_ld();
          const float* dpv = reinterpret_cast<const float*>(&dr[0][0]);
          uint32_t dk[32];
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float4 d4 = dv4[e2];
            const uint32_t w0 = pk[2 * e2], w1 = pk[2 * e2 + 1];
            dk[2 * e2] = pack_bf16x2(bf16lo(w0) * (dpv[4 * e2 + 0] - d4.x), bf16hi(w0) * (dpv[4 * e2 + 1] - d4.y));
            dk[2 * e2 + 1] = pack_bf16x2(bf16lo(w1) * (dpv[4 * e2 + 2] - d4.z), bf16hi(w1) * (dpv[4 * e2 + 3] - d4.w));
          }
          tmem_st32(tmem + L::kTmDP + lane_off + h * 64, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR_DSF);
      }
      u += static_cast<uint32_t>(it.n);
      // ---- epilogue: dK (times scale) and dV rows of this key tile; a key
      // tile that no query sees gets zeros
      const bool have = ok && it.n > 0;
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(BAR_ACC, static_cast<uint32_t>(qi) & 1u, a.status, abort_flag));
        tc_fence_after();
      }
      // TMEM loads are warp-collective: every lane loads, only rows < Nkv store
      const bool store = key < a.Nkv;
      const size_t orow = (static_cast<size_t>(it.b) * a.Hkv + it.hkv) * a.Nkv + (store ? key : 0);
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        // this warpgroup's half of the row: columns [h D/2, (h+1) D/2)
        __nv_bfloat16* dst_row = (which ? a.dv : a.dk) + orow * D + h * (D / 2);
        const float mul = which ? 1.f : a.scale;
        const uint32_t src = tmem + (which ? L::kTmDV : L::kTmDK) + lane_off + h * (D / 2);
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v[32];
          if (have && ok) {
            tmem_ld32(src + c * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * mul, __uint_as_float(v[8 * e + 1]) * mul);
              w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * mul, __uint_as_float(v[8 * e + 3]) * mul);
              w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * mul, __uint_as_float(v[8 * e + 5]) * mul);
              w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * mul, __uint_as_float(v[8 * e + 7]) * mul);
              dst[e] = w;
            }
          }
        }
      }
      if (it.n > 0) {
        // dV and dK have been read: the next key tile's first products may overwrite them
        tc_fence_before();
        mbar_arrive(BAR_ACCE);
        ++qi;
      }
      if (!ok) break;
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag)))) break;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      mbar_arrive(BAR_ITE(sl));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dQ: work items are (query tile, batch, query head), later query tiles
// first.  A CTA runs its own item and then takes over the items of CTAs not
// yet launched (cluster launch control: a successful try_cancel hands over
// the cancelled CTA's index).  Its K/V ring and its S, dP and dS hand-offs
// run on across items as one stream of key tiles: the next item's Q and dO
// load as soon as the current item's last S and dP are issued, and the next
// item's first S and dP follow the current item's last dQ product while the
// work warps write that dQ out.  That overlaps each item's fixed cost (Q/dO
// load latency, first products, dQ epilogue, CTA launch) with work.
// ---------------------------------------------------------------------------
template <int D>
struct DqLayout {
  using T = BwdTiles<D>;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + T::kTileBytes;
  // K_j is read by S_j and again by dQ_j, so its slot frees late: three K
  // slots let K_{j+1} load while dQ_{j-1} still runs.  V_j is read by dP_j only.
  static constexpr int kSK = 3, kSV = 2;
  static constexpr int kK = kDO + T::kTileBytes;
  static constexpr int kV = kK + kSK * T::kTileBytes;
  static constexpr int kBar = kV + kSV * T::kTileBytes;
  // q_full, q_empty, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full, loaded, dp_full, ds_full,
  // ds_empty, acc_done, dq_empty, item_full[2], item_empty[2], fin
  static constexpr int kNumBars = 2 + 2 * kSK + 2 * kSV + 7 + 4 + 1;
  static constexpr int kResp = (kBar + kNumBars * 8 + 15) & ~15;   // two 16-byte work-request answers
  static constexpr int kMisc = kResp + 32;
  static constexpr int kAlloc = kMisc + 16 + 1024;
  static_assert(kAlloc <= 232448, "dynamic shared memory per block");
  // TMEM: S | dP | dQ | dS (bf16, 64 columns)
  static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDQ = 256, kTmDS = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
};

// Key tiles query tile [q0, q0 + 128) must visit (0 if no row sees a key).
__host__ __device__ inline int key_tiles_for(int q0, const BwdArgs& a) {
  int kv_end = a.Nkv;
  if (a.causal) kv_end = min(a.Nkv, min(q0 + kT, a.Nq) - 1 + (a.Nkv - a.Nq) + 1);
  return kv_end <= 0 ? 0 : (kv_end + kT - 1) / kT;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdArgs a) {
  using T = BwdTiles<D>;
  using L = DqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQ = sb + L::kQ, sDO = sb + L::kDO, sK = sb + L::kK, sV = sb + L::kV;
  const uint32_t bar0 = sb + L::kBar;
  constexpr int kSK = L::kSK, kSV = L::kSV;
  // q_empty: the item's last S and dP have read Q and dO
  const uint32_t BAR_Q = bar0, BAR_QE = bar0 + 8u;
  auto BAR_KF = [&](int s) { return bar0 + 8u * (2 + s); };
  auto BAR_KE = [&](int s) { return bar0 + 8u * (2 + kSK + s); };
  auto BAR_VF = [&](int s) { return bar0 + 8u * (2 + 2 * kSK + s); };
  auto BAR_VE = [&](int s) { return bar0 + 8u * (2 + 2 * kSK + kSV + s); };
  // loaded: S and dP of the current tile are in registers (both buffers may be
  // overwritten); ds_empty: the dQ product has read the dS buffer; dq_empty:
  // the epilogue has read the dQ accumulator; item_full / item_empty: a work
  // request's answer has landed / has been read by every consumer
  const uint32_t bar1 = bar0 + 8u * (2 + 2 * kSK + 2 * kSV);
  const uint32_t BAR_SF = bar1, BAR_LOADED = bar1 + 8u, BAR_DPF = bar1 + 16u, BAR_DSF = bar1 + 24u,
                 BAR_DSE = bar1 + 32u, BAR_ACC = bar1 + 40u, BAR_DQE = bar1 + 48u, BAR_FIN = bar1 + 88u;
  auto BAR_ITF = [&](int s) { return bar1 + 56u + 8u * s; };
  auto BAR_ITE = [&](int s) { return bar1 + 72u + 8u * s; };
  const uint32_t sResp = sb + L::kResp;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  struct Item {
    int b, hq, hkv, bh, q0, n;
  };
  const int bh_count = a.B * a.Hq;
  auto decode_item = [&](int idx) {
    Item it;
    const int grp = idx / (a.q_group * a.n_qt), base = grp * a.q_group;
    const int in_grp = min(a.q_group, bh_count - base), rem = idx - grp * a.q_group * a.n_qt;
    it.bh = base + rem % in_grp;
    it.b = it.bh / a.Hq;
    it.hq = it.bh % a.Hq;
    it.hkv = it.hq / (a.Hq / a.Hkv);
    it.q0 = (a.n_qt - 1 - rem / in_grp) * kT;
    it.n = key_tiles_for(it.q0, a);
    return it;
  };
  // Work request k >= 1 (the item after the k-th) answers in slot k & 1; it is
  // that slot's ((k - 1) >> 1)-th use.
  auto resp_parity = [](int k) { return static_cast<uint32_t>((k - 1) >> 1) & 1u; };

  if (threadIdx.x == 0) {
    mbar_init(BAR_Q, 1);
    mbar_init(BAR_QE, 1);
    for (int s = 0; s < kSK; ++s) {
      mbar_init(BAR_KF(s), 1);
      mbar_init(BAR_KE(s), 1);
    }
    for (int s = 0; s < kSV; ++s) {
      mbar_init(BAR_VF(s), 1);
      mbar_init(BAR_VE(s), 1);
    }
    mbar_init(BAR_SF, 1);
    mbar_init(BAR_LOADED, 256);
    mbar_init(BAR_DPF, 1);
    mbar_init(BAR_DSF, 256);
    mbar_init(BAR_DSE, 1);
    mbar_init(BAR_ACC, 1);
    mbar_init(BAR_DQE, 256);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR_ITF(s), 1);
      mbar_init(BAR_ITE(s), 1 + 256);   // the MMA warp's leader and every work thread
    }
    mbar_init(BAR_FIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < kWorkWarp0) {
  setmaxnreg_dec<kBwdRegsControl>();
  if (warp == 0 && lane == 0) {
    // ======================= TMA producer =======================
    bool ok = true;
    uint32_t gk = 0, gv = 0;   // K and V tiles loaded so far: ring slot g % slots, use g / slots
    int qi = 0;                // items whose Q and dO were loaded
    int requested = 0, answered = 0;
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0 && ok; ++k) {
      // ask for the item after this one now, so the answer is back when it is needed
      {
        const int kn = k + 1, sl = kn & 1;
        if (kn >= 3 && !(ok = mbar_wait(BAR_ITE(sl), resp_parity(kn - 2), a.status, abort_flag))) break;
        fence_proxy_async_smem();   // the slot's previous answer was read through the generic proxy
        mbar_arrive_expect_tx(BAR_ITF(sl), 16);
        clc_try_cancel(sResp + 16 * sl, BAR_ITF(sl));
        requested = kn;
      }
      const Item it = decode_item(idx);
      if (it.n > 0) {
        // the Q/dO buffer is free once the previous item's last S and dP completed
        if (qi > 0 && !(ok = mbar_wait(BAR_QE, static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag))) break;
        const int zq = it.b * a.Hq + it.hq, zk = it.b * a.Hkv + it.hkv;
        mbar_arrive_expect_tx(BAR_Q, 2 * T::kTileBytes);
        tma_load_4d(sQ, &tmQ, BAR_Q, 0, it.q0, 0, zq);
        tma_load_4d(sDO, &tmDO, BAR_Q, 0, it.q0, 0, zq);
        ++qi;
        for (int j = 0; j < it.n; ++j) {
          const int sk = static_cast<int>(gk % kSK), sv = static_cast<int>(gv % kSV);
          if (!(ok = mbar_wait(BAR_KE(sk), ((gk / kSK) & 1u) ^ 1u, a.status, abort_flag))) break;
          mbar_arrive_expect_tx(BAR_KF(sk), T::kTileBytes);
          tma_load_4d(sK + sk * T::kTileBytes, &tmK, BAR_KF(sk), 0, j * kT, 0, zk);
          ++gk;
          if (!(ok = mbar_wait(BAR_VE(sv), ((gv / kSV) & 1u) ^ 1u, a.status, abort_flag))) break;
          mbar_arrive_expect_tx(BAR_VF(sv), T::kTileBytes);
          tma_load_4d(sV + sv * T::kTileBytes, &tmV, BAR_VF(sv), 0, j * kT, 0, zk);
          ++gv;
        }
        if (!ok) break;
      }
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
      answered = kn;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
    }
    // drain: no copy into this CTA's shared memory may still be in flight at exit
    if (answered < requested)
      mbar_wait(BAR_ITF(requested & 1), resp_parity(requested), nullptr, nullptr, kWaitLimitNs);
    if (qi > 0) mbar_wait(BAR_Q, static_cast<uint32_t>(qi - 1) & 1u, nullptr, nullptr, kWaitLimitNs);
    for (uint32_t g = (gk > static_cast<uint32_t>(kSK) ? gk - kSK : 0u); g < gk; ++g)
      mbar_wait(BAR_KF(static_cast<int>(g % kSK)), (g / kSK) & 1u, nullptr, nullptr, kWaitLimitNs);
    for (uint32_t g = (gv > static_cast<uint32_t>(kSV) ? gv - kSV : 0u); g < gv; ++g)
      mbar_wait(BAR_VF(static_cast<int>(g % kSV)), (g / kSV) & 1u, nullptr, nullptr, kWaitLimitNs);
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    // The whole warp runs the issue loop (warp-uniform descriptors and
    // waits); the elected lane issues the MMAs and their commits.
    const bool leader = elect_one_sync();
    auto commit = [&](uint32_t bar) {
      if (leader) mma_commit(bar);
      __syncwarp();
    };
    constexpr uint32_t idesc_s = idesc_bf16_f32(kT, kT, false);
    constexpr uint32_t idesc_acc = idesc_bf16_f32(kT, D, true);
    const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024), dDO = smem_desc_sw128(sDO, 16, 1024);
    const uint64_t dKk = smem_desc_sw128(sK, 16, 1024), dVk = smem_desc_sw128(sV, 16, 1024);
    const uint64_t dKm = smem_desc_sw128(sK, T::kChunkBytes, 1024);
    constexpr uint64_t kStep = T::kTileBytes >> 4;
    // S = Q K^T and dP = dO V^T of the key tile in ring positions (gkk, gvv)
    auto issue_s_dp = [&](uint32_t gkk, uint32_t gvv) -> bool {
      const int sk = static_cast<int>(gkk % kSK), sv = static_cast<int>(gvv % kSV);
      if (!mbar_wait_warp(BAR_KF(sk), (gkk / kSK) & 1u, a.status, abort_flag)) return false;
      tc_fence_after();
      mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmS, dQ, dKk + sk * kStep, idesc_s);
      commit(BAR_SF);
      if (!mbar_wait_warp(BAR_VF(sv), (gvv / kSV) & 1u, a.status, abort_flag)) return false;
      tc_fence_after();
      mma_kmajor_tile<T::kChunks>(leader, tmem + L::kTmDP, dDO, dVk + sv * kStep, idesc_s);
      commit(BAR_DPF);
      commit(BAR_VE(sv));   // V_j is read by dP_j only
      return true;
    };
    bool ok = true;
    uint32_t t = 0;            // key tiles of this CTA so far (S/dP/dS hand-off phases)
    uint32_t gk = 0, gv = 0;   // K/V ring positions, as the producer's
    int qi = 0;                // items with keys so far
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0 && ok; ++k) {
      const Item it = decode_item(idx);
      if (it.n > 0) {
        // the first tile's S and dP: the previous tile's are in registers and
        // this item's Q and dO have landed
        if (t > 0 && !(ok = mbar_wait_warp(BAR_LOADED, (t - 1) & 1u, a.status, abort_flag))) break;
        if (!(ok = mbar_wait_warp(BAR_Q, static_cast<uint32_t>(qi) & 1u, a.status, abort_flag))) break;
        if (!(ok = issue_s_dp(gk, gv))) break;
        if (it.n == 1) commit(BAR_QE);
        for (int j = 0; j < it.n; ++j) {
          const uint32_t tj = t + static_cast<uint32_t>(j), gkj = gk + static_cast<uint32_t>(j);
          // next S and dP as soon as the work warps hold this tile's in registers
          if (j + 1 < it.n) {
            if (!(ok = mbar_wait_warp(BAR_LOADED, tj & 1u, a.status, abort_flag))) break;
            if (!(ok = issue_s_dp(gkj + 1, gv + static_cast<uint32_t>(j) + 1))) break;
            if (j + 2 == it.n) commit(BAR_QE);   // the item's last S and dP: Q and dO are free
          }
          // dQ += dS K_j once dS is in its buffer; an item's first product
          // overwrites the accumulator, which the previous epilogue must have read
          if (!(ok = mbar_wait_warp(BAR_DSF, tj & 1u, a.status, abort_flag))) break;
          if (j == 0 && qi > 0 &&
              !(ok = mbar_wait_warp(BAR_DQE, static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag)))
            break;
          tc_fence_after();
          const int sk = static_cast<int>(gkj % kSK);
          mma_tmem_a(leader, tmem + L::kTmDQ, tmem + L::kTmDS, tmem + L::kTmDS + 32, dKm + sk * kStep, idesc_acc,
                     j > 0);
          commit(BAR_DSE);
          commit(BAR_KE(sk));   // K_j is read by S_j and dQ_j
        }
        if (!ok) break;
        commit(BAR_ACC);
        t += static_cast<uint32_t>(it.n);
        gk += static_cast<uint32_t>(it.n);
        gv += static_cast<uint32_t>(it.n);
        ++qi;
      }
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = mbar_wait_warp(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      __syncwarp();
      if (leader) mbar_arrive(BAR_ITE(sl));
    }
    // no commit may still be pending when the CTA exits
    commit(BAR_FIN);
    mbar_wait_warp(BAR_FIN, 0, nullptr, nullptr);
  }
  } else {
    setmaxnreg_inc<kBwdRegsWork>();
    // ======================= per-query-row work + epilogue =======================
    const int h = (warp - kWorkWarp0) / 4;         // key columns [64h, 64h + 64) of each tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c2 = a.scale_log2;
    bool ok = true;
    uint32_t t = 0;   // key tiles of this CTA so far
    int qi = 0;       // items with keys so far
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0; ++k) {
      const Item it = decode_item(idx);
      const int q0 = it.q0, n = it.n;
      const int qrow = q0 + r;
      const size_t vrow = static_cast<size_t>(it.bh) * (a.n_qt * kT) + qrow;   // padded rows exist for every r
      const float l2 = a.lse2[vrow], dl = a.delta[vrow];
      const int vis_end = a.causal ? min(a.Nkv, qrow + (a.Nkv - a.Nq) + 1) : a.Nkv;
      for (int j = 0; j < n && ok; ++j) {
        const uint32_t tj = t + static_cast<uint32_t>(j);
        const uint32_t ph = tj & 1u;
        ok = mbar_wait(BAR_SF, ph, a.status, abort_flag);
        ok = ok && mbar_wait(BAR_DPF, ph, a.status, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int lim = vis_end - j * kT - h * 64;   // visible key columns of this half: [0, lim)
        const bool need_mask = (j * kT + kT > a.Nkv) || (a.causal && j * kT + kT - 1 > q0 + (a.Nkv - a.Nq));
        uint32_t pk[32];
        {
          uint32_t sr[2][32], dr[2][32];
          tmem_ld32(tmem + L::kTmS + lane_off + h * 64, sr[0]);
          tmem_ld32(tmem + L::kTmS + lane_off + h * 64 + 32, sr[1]);
          tmem_ld32(tmem + L::kTmDP + lane_off + h * 64, dr[0]);
          tmem_ld32(tmem + L::kTmDP + lane_off + h * 64 + 32, dr[1]);
          tmem_wait_ld();
          // this half of S and dP is in registers: the next tile's products may
          // overwrite both buffers once the other half has read its part too
          tc_fence_before();
          mbar_arrive(BAR_LOADED);
          const float* sv = reinterpret_cast<const float*>(&sr[0][0]);
          const float* dpv = reinterpret_cast<const float*>(&dr[0][0]);
          if (need_mask)   // uniform across the CTA
            ds_row_half<true>(sv, dpv, c2, l2, dl, lim, pk);
          else
            ds_row_half<false>(sv, dpv, c2, l2, dl, lim, pk);
        }
        // the previous dQ product (of this or an earlier item) must have read the dS buffer
        if (tj > 0) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR_DSE, (tj - 1) & 1u, a.status, abort_flag)))) break;
          tc_fence_after();
        }
        tmem_st32(tmem + L::kTmDS + lane_off + h * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR_DSF);
      }
      t += static_cast<uint32_t>(n);
      // ---- epilogue: dQ (times scale); a query tile that sees no key gets zeros
      const bool have = ok && n > 0;
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(BAR_ACC, static_cast<uint32_t>(qi) & 1u, a.status, abort_flag));
        tc_fence_after();
      }
      // TMEM loads are warp-collective: every lane loads, only rows < Nq store
      const bool store = qrow < a.Nq;
      // this warpgroup's half of the row: columns [h D/2, (h+1) D/2)
      __nv_bfloat16* dst_row = a.dq + (static_cast<size_t>(it.bh) * a.Nq + (store ? qrow : 0)) * D + h * (D / 2);
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t v[32];
        if (have && ok) {
          tmem_ld32(tmem + L::kTmDQ + lane_off + h * (D / 2) + c * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * a.scale, __uint_as_float(v[8 * e + 1]) * a.scale);
            w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * a.scale, __uint_as_float(v[8 * e + 3]) * a.scale);
            w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * a.scale, __uint_as_float(v[8 * e + 5]) * a.scale);
            w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * a.scale, __uint_as_float(v[8 * e + 7]) * a.scale);
            dst[e] = w;
          }
        }
      }
      if (n > 0) {
        // the accumulator has been read: the next item's first dQ product may overwrite it
        tc_fence_before();
        mbar_arrive(BAR_DQE);
        ++qi;
      }
      if (!ok) break;
      // the next item (or none)
      const int kn = k + 1, sl = kn & 1;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag)))) break;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      mbar_arrive(BAR_ITE(sl));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

template <int D>
ta_status launch_bwd_d(const void* q, const void* k, const void* v, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                       int Nq, int Nkv, float scale, int causal, cudaStream_t stream) {
  BwdArgs a;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.n_qt = (Nq + kT - 1) / kT;
  a.n_kt = (Nkv + kT - 1) / kT;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  const size_t padded = static_cast<size_t>(B) * Hq * a.n_qt * kT;
  float* ws = static_cast<float*>(workspace);
  a.delta = ws;
  a.lse2 = ws + padded;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  {
    // Heads per launch group.  L2 bound: ~24 MB of streamed operand (dK/dV: a
    // KV head's query heads' Q and dO; dQ: a query head's K and V).  Balance
    // bound: a group's work at least 2 x SMs x its heaviest item, so the
    // heaviest items of the last group still start early (with one GQA KV
    // head per group the causal backward ran 12% slower; factors 1.5 and 3
    // measured slower than 2).  The balance bound wins; groups are then made
    // near equal.  Causal workload: 3 groups of ~22 heads, 0.898 -> 0.863 ms,
    // DRAM traffic 2.05 -> 0.70 GB per call.
    int sms = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0) {
      cudaGetLastError();
      sms = 148;
    }
    constexpr double kGroupBytes = 24.0 * (1 << 20);
    auto group_size = [&](int count, double stream_bytes, double heaviest, double per_head) {
      if (count <= 0 || per_head <= 0) return 1;
      const int by_l2 = std::max(1, static_cast<int>(kGroupBytes / std::max(stream_bytes, 1.0)));
      const int by_balance = static_cast<int>(std::ceil(2.0 * sms * heaviest / per_head));
      const int g = std::min(count, std::max(by_l2, by_balance));
      const int n_groups = std::max(1, count / g);
      return (count + n_groups - 1) / n_groups;
    };
    const int G = Hq / Hkv;
    double kv_work = 0, kv_max = 0, q_work = 0, q_max = 0;
    for (int kt = 0; kt < a.n_kt; ++kt) {
      const int i0 = first_query_tile(kt, a);
      const double w = static_cast<double>(G) * (i0 < a.n_qt ? a.n_qt - i0 : 0);
      kv_work += w;
      kv_max = std::max(kv_max, w);
    }
    for (int qt = 0; qt < a.n_qt; ++qt) {
      const double w = key_tiles_for(qt * kT, a);
      q_work += w;
      q_max = std::max(q_max, w);
    }
    a.kv_group = group_size(B * Hkv, static_cast<double>(G) * Nq * D * 2 * 2, kv_max, kv_work);
    a.q_group = group_size(B * Hq, static_cast<double>(Nkv) * D * 2 * 2, q_max, q_work);
  }
  a.status = device_status_ptr();
  if (!a.status) return fail(TA_ERR_CUDA, "attn_bwd: device status word");

  // delta and lse2 for every padded query row
  {
    const long long threads = static_cast<long long>(padded) * 8;
    bwd_prep_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, ws, ws + padded, Nq,
        a.n_qt * kT, static_cast<long long>(padded));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(TA_ERR_CUDA, "attn_bwd: prep launch", e);
  }
  CUtensorMap tq, tk, tv, tdo;
  ta_status st;
  if ((st = encode_rows_chunked(&tq, q, D, Nq, B * Hq)) != TA_OK) return st;
  if ((st = encode_rows_chunked(&tdo, dout, D, Nq, B * Hq)) != TA_OK) return st;
  if ((st = encode_rows_chunked(&tk, k, D, Nkv, B * Hkv)) != TA_OK) return st;
  if ((st = encode_rows_chunked(&tv, v, D, Nkv, B * Hkv)) != TA_OK) return st;
  static int done_kv[64] = {0}, done_q[64] = {0};
  cudaError_t e = ensure_smem_limit(bwd_dkdv_kernel<D>, DkdvLayout<D>::kAlloc, done_kv);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "attn_bwd: shared-memory limit (dK/dV)", e);
  e = ensure_smem_limit(bwd_dq_kernel<D>, DqLayout<D>::kAlloc, done_q);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "attn_bwd: shared-memory limit (dQ)", e);
  const unsigned grid_kv = static_cast<unsigned>(a.n_kt) * static_cast<unsigned>(B * Hkv);
  bwd_dkdv_kernel<D><<<grid_kv, kBwdThreads, DkdvLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return fail(TA_ERR_CUDA, "attn_bwd: dK/dV launch", e);
  const unsigned grid_q = static_cast<unsigned>(a.n_qt) * static_cast<unsigned>(B * Hq);
  {
    // Programmatic stream serialization: the dQ kernel reads only what the
    // prep kernel wrote (finished before the dK/dV kernel began), so its CTAs
    // may start on the SMs the dK/dV kernel's CTAs free while its last items
    // run (the dK/dV CTAs signal dependents as they start).  Causal backward
    // 0.858 -> 0.851 ms; gradients bitwise unchanged.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_q);
    cfg.blockDim = dim3(kBwdThreads);
    cfg.dynamicSmemBytes = DqLayout<D>::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, bwd_dq_kernel<D>, tq, tk, tv, tdo, a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return fail(TA_ERR_CUDA, "attn_bwd: dQ launch", e);
  return TA_OK;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int Hq, int Nq) {
  const size_t padded = static_cast<size_t>(B) * Hq * ((Nq + kT - 1) / kT) * kT;
  return ((2 * padded * sizeof(float)) + 255) & ~size_t(255);
}

ta_status launch_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                          const float* lse, void* dq, void* dk, void* dv, void* workspace, int B, int Hq, int Hkv,
                          int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  if (d == 128)
    return launch_bwd_d<128>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nkv, scale, causal,
                             stream);
  return launch_bwd_d<64>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
}

}  // namespace ta
