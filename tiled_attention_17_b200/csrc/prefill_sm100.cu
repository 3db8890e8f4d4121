// Fused, tiled attention forward for sm_100a (B200).
//
// O = softmax(scale * Q K^T [+ causal mask]) V computed in one pass over K/V
// tiles with the online-softmax recurrence, so the score and probability
// tiles live only in tensor memory and registers and never reach HBM
// (Gemini 3 Flash kernel-fusion post, sections 1-3; FlashAttention
// optimisation article, sections 3.1-3.2 and 7.1).
//
// Work item = two 128-row query tiles sharing one K/V stream (two tiles of one
// head, or one tile of two GQA heads).  Dense and FP8 CTAs are persistent: after
// their own item they take over the items of CTAs not yet launched (cluster
// launch control), so the next item's loads and first Q.K^T overlap the
// epilogue of the current one.  Instantiations: dense [B, H, N, d] bf16; FP8
// (kFp8) E4M3 inputs; (kPaged) varlen query rows packed as [total_q, Hq, d]
// against K/V gathered page by page from a paged cache through a block table
// (chunked prefill, LLM-inference article section 3.2; PagedAttention,
// GPU-optimisation tag page).  Warp roles (384 threads, three warpgroups):
//   warp 0      TMA producer: Q tiles once per item, then K_j / V_j into a
//               smem ring; makes the work requests
//   warp 1      TMEM allocator + tcgen05.mma issuer (whole warp, one elected
//               lane issues)
//   warps 2-3   idle after setup
//   warps 4-7   softmax warpgroup for query tile 0 (one thread per row)
//   warps 8-11  softmax warpgroup for query tile 1
// The block launches at 168 registers per thread (the per-sub-partition
// register file holds three warps of that size); the first warpgroup then
// releases registers (setmaxnreg.dec to 56) and the softmax warpgroups take
// them (setmaxnreg.inc to 224): 128*56 + 256*224 = 384*168.
// Tensor memory (512 columns): S0 | S1 | O0 | O1.  P (bf16) overwrites the
// first half of its S tile and feeds the P.V product straight from TMEM.
//
// Per K/V tile j the MMA issue order is
//   O0 += P0 V_j ; S0 = Q0 K_{j+1}^T ; O1 += P1 V_j ; S1 = Q1 K_{j+1}^T
// so each softmax warpgroup works while the tensor pipe serves the other tile.
// Softmax follows the recurrence of the article's section 3.2.1: running max
// m and sum l per row, e^(m_old - m_new) rescaling of l and of the partial O.
// The O rescale is skipped while the max has not grown by more than 2^8 in
// exp2 units (the page's "rescale only when the max changes", with a margin);
// the result is unchanged because numerator and denominator share the stale
// max.  lse = m * scale + ln(l) is written per row (the row max and
// normaliser kept for a recomputing backward, kernel-fusion post section 4).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "tiledattn_internal.h"

namespace ta {

constexpr int kBM = 128;      // query rows per tile
constexpr int kBN = 128;      // keys per tile
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kLaunchRegs = 168;     // what ptxas must report for this kernel
constexpr int kRegsControl = 56;     // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsSoftmax = 224;    // warpgroups 1-2 after setmaxnreg.inc
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * kLaunchRegs, "register split");
static_assert(kRegsControl + 2 * kRegsSoftmax <= 512, "per sub-partition: one warp of each warpgroup");
constexpr float kRescaleLog2 = 8.0f;   // skip O rescale while max grew by <= 2^8
// Column pairs whose index i has bit (i % 8) set in the mask compute 2^x on
// the FMA pipe (exp2_poly2) instead of the MUFU unit.  bf16: moving 1/8 to 4/8
// of them there was measured, none was faster on B200, so all stay on MUFU.
// fp8: the products take half the tensor cycles and MUFU limits more.  With
// the current issue loop and persistent CTAs, 1/8 (pair 0 of every 8) is
// fastest: +3% over none and over 3/8 (2/8: +1.5%, 4/8: -4%, 6/8: -13%).
constexpr unsigned kPolyMask = 0x00u;
constexpr unsigned kPolyMaskFp8 = 0x01u;

template <int D, bool kFp8 = false>
struct PrefillLayout {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!kFp8 || D == 128, "fp8 inputs: d = 128 (one 128-byte swizzle row)");
  static constexpr int kElemBytes = kFp8 ? 1 : 2;
  static constexpr int kChunkElems = 128 / kElemBytes;           // elements of one 128-byte swizzle row
  static constexpr int kChunks = D / kChunkElems;                // swizzle atoms along d
  static constexpr int kTileBytes = 128 * D * kElemBytes;        // one 128-row tile
  static constexpr int kChunkBytes = 128 * 128;                  // 128 rows x 128 bytes
  static constexpr int kStages = (kTileBytes > kChunkBytes) ? 2 : 3;  // K ring and V ring depth
  static constexpr int kKeysPerMma = 32 / kElemBytes;            // one MMA reads 32 bytes of each row
  static constexpr int kPWords = 64 * kElemBytes / 4;            // TMEM columns of one half (64 keys) of P
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // barriers: q, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_ready[2], o_done[2],
  // p_half[2] (first 64 keys of P written), item_full[2], item_empty[2] (work-request
  // responses), q_free, o_free[2] (epilogue has read O), mma_done
  static constexpr int kNumBars = 1 + 4 * kStages + 16;
  static constexpr int kResp = (kBar + kNumBars * 8 + 15) & ~15;   // two 16-byte work-request responses
  static constexpr int kMisc = kResp + 32;            // tmem base (4 B) + abort flag (4 B)
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;        // slack to align the base to 1024 B
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO0 = 256, kTmO1 = 256 + D;
};

struct PrefillArgs {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nkv;
  int n_units;       // work units along the queries: ceil(Nq / 256) pairs, or ceil(Nq / 128) tiles (head_pair)
  int head_pair;     // 1: a CTA takes one 128-row tile of two query heads sharing a KV head (GQA, even group)
  int causal;
  float scale;       // natural-log scale (for lse)
  float scale_log2;  // scale * log2(e)
  unsigned* status;
  // varlen prefill over the paged cache (kPaged): the queries of num_seqs
  // sequences are packed as [total_q, Hq, d] (o and lse the same way), and
  // sequence s owns rows [cu_seqlens[s], cu_seqlens[s+1]) and seq_lens[s] keys
  const int32_t* block_table;
  const int32_t* cu_seqlens;
  const int32_t* seq_lens;
  int num_seqs, total_q, max_q_len, page_size, max_pages, num_pages_total;
  // fp8 inputs: the values are descale * e4m3(code); q and k descales are
  // folded into scale / scale_log2, v's is applied to O in the epilogue
  float v_descale;
};

// Number of K/V tiles query tile [q0, q0+128) must visit (0 if it has no rows
// or every row is fully masked).
__device__ __forceinline__ int kv_tiles_for(int q0, int Nq, int Nkv, int causal) {
  if (q0 >= Nq) return 0;
  int kv_end = Nkv;
  if (causal) {
    int last = min(q0 + kBM, Nq) - 1;
    kv_end = min(Nkv, last + (Nkv - Nq) + 1);
  }
  return kv_end <= 0 ? 0 : (kv_end + kBN - 1) / kBN;
}

template <int D, bool kPaged, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
  static_assert(!(kPaged && kFp8), "fp8 inputs: dense layout only");
  using L = PrefillLayout<D, kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ, sK = sbase + L::kK, sV = sbase + L::kV;
  const uint32_t bar0 = sbase + L::kBar;
  auto BAR_Q = [&]() { return bar0; };
  auto BAR_KF = [&](int s) { return bar0 + 8u * (1 + s); };
  auto BAR_KE = [&](int s) { return bar0 + 8u * (1 + L::kStages + s); };
  auto BAR_VF = [&](int s) { return bar0 + 8u * (1 + 2 * L::kStages + s); };
  auto BAR_VE = [&](int s) { return bar0 + 8u * (1 + 3 * L::kStages + s); };
  auto BAR_SF = [&](int t) { return bar0 + 8u * (1 + 4 * L::kStages + t); };
  auto BAR_PR = [&](int t) { return bar0 + 8u * (3 + 4 * L::kStages + t); };
  auto BAR_OD = [&](int t) { return bar0 + 8u * (5 + 4 * L::kStages + t); };
  auto BAR_PH = [&](int t) { return bar0 + 8u * (7 + 4 * L::kStages + t); };
  auto BAR_ITF = [&](int s) { return bar0 + 8u * (9 + 4 * L::kStages + s); };
  auto BAR_ITE = [&](int s) { return bar0 + 8u * (11 + 4 * L::kStages + s); };
  auto BAR_QE = [&]() { return bar0 + 8u * (13 + 4 * L::kStages); };
  auto BAR_OF = [&](int t) { return bar0 + 8u * (14 + 4 * L::kStages + t); };
  auto BAR_FIN = [&]() { return bar0 + 8u * (16 + 4 * L::kStages); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work items.  A CTA starts with item blockIdx.x and then takes over
  // the items of CTAs that have not launched yet (cluster launch control: a
  // successful try_cancel hands over the cancelled CTA's index).  Each SM so
  // runs a sequence of items in launch order, heaviest first, and the next
  // item's loads and first product overlap the current item's epilogue.  An
  // item's two 128-row query tiles are two consecutive tiles of one head, or
  // (head_pair) the same tile of two query heads of one GQA group: both read
  // the same K/V stream.  Dense: (unit, batch, head[s]).  Paged: (unit,
  // sequence, head[s]), with the sequence's query and key counts read (and
  // range-checked) here; units past a sequence's queries are empty items.
  struct Item {
    int b, hq_0, hq_1, hkv, Nq, Nkv, q_base, q0_0, q0_1, nt_0, nt_1, n_max;
    bool valid;
  };
  auto decode_item = [&](int idx, bool report) {
    Item it;
    const int heads_per_item = a.head_pair ? 2 : 1;
    const int hx_count = a.Hq / heads_per_item;
    const int bh_count = (kPaged ? a.num_seqs : a.B) * hx_count;
    // Dense: query units heaviest first across all heads (causal balance).
    // Paged: stream-major, all units of one (sequence, head[s]) adjacent,
    // heaviest first, so the CTAs running at once share one sequence's K/V
    // in L2 (DRAM traffic 5.1 -> 1.1 GB on the chunked-prefill mix, about
    // the algorithmic minimum) and its empty units come first and exit.
    const int unit = kPaged ? a.n_units - 1 - idx % a.n_units : a.n_units - 1 - idx / bh_count;
    const int bh = kPaged ? idx / a.n_units : idx % bh_count;
    it.b = bh / hx_count;                             // sequence when paged
    it.hq_0 = (bh % hx_count) * heads_per_item;      // query head of tile 0
    it.hq_1 = it.hq_0 + heads_per_item - 1;          // query head of tile 1
    it.hkv = it.hq_0 / (a.Hq / a.Hkv);
    it.Nq = a.Nq;
    it.Nkv = a.Nkv;
    it.q_base = 0;                                   // packed row of the sequence's first query (paged)
    if constexpr (kPaged) {
      int lo = a.cu_seqlens[it.b], hi = a.cu_seqlens[it.b + 1];
      int len = a.seq_lens[it.b];
      unsigned bad = 0;
      if (lo < 0 || lo > a.total_q || hi < lo || hi > a.total_q || hi - lo > a.max_q_len) bad |= kDevBadSeqLen;
      if (len < 0 || len > a.max_pages * a.page_size) bad |= kDevBadSeqLen;
      lo = min(max(lo, 0), a.total_q);
      hi = min(max(hi, lo), min(a.total_q, lo + a.max_q_len));
      len = min(max(len, 0), a.max_pages * a.page_size);
      if (bad && report && unit == 0 && it.hq_0 == 0) atomicOr(a.status, bad);
      it.q_base = lo;
      it.Nq = hi - lo;
      it.Nkv = len;
    }
    it.q0_0 = a.head_pair ? unit * kBM : unit * 2 * kBM;
    it.q0_1 = a.head_pair ? it.q0_0 : it.q0_0 + kBM;
    it.valid = !(kPaged && it.q0_0 >= it.Nq);
    it.nt_0 = it.valid ? kv_tiles_for(it.q0_0, it.Nq, it.Nkv, a.causal) : 0;
    it.nt_1 = it.valid ? kv_tiles_for(it.q0_1, it.Nq, it.Nkv, a.causal) : 0;
    it.n_max = max(it.nt_0, it.nt_1);
    return it;
  };
  // Dense and FP8 CTAs take further items; a paged CTA runs its own item
  // only (about half of a varlen grid are empty units past their sequence's
  // queries, which exit at once instead of costing a work request each).
  constexpr bool kPersistent = !kPaged;
  if constexpr (!kPersistent) {
    if (!decode_item(static_cast<int>(blockIdx.x), false).valid) return;   // uniform per CTA
  }
  // Work request k >= 1 (the item after the k-th) answers in slot k & 1; it is
  // that slot's ((k - 1) >> 1)-th use.
  const uint32_t sResp = sbase + L::kResp;
  auto resp_parity = [](int k) { return static_cast<uint32_t>((k - 1) >> 1) & 1u; };

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(BAR_Q(), 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(BAR_KF(s), 1);
      mbar_init(BAR_KE(s), 1);
      mbar_init(BAR_VF(s), 1);
      mbar_init(BAR_VE(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(BAR_SF(t), 1);
      mbar_init(BAR_PR(t), 128);
      mbar_init(BAR_OD(t), 1);
      mbar_init(BAR_PH(t), 128);
      mbar_init(BAR_ITF(t), 1);
      mbar_init(BAR_ITE(t), 1 + 256);   // the MMA warp's leader and every softmax thread
      mbar_init(BAR_OF(t), 128);
    }
    mbar_init(BAR_QE(), 1);
    mbar_init(BAR_FIN(), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0 && lane == 0) {
    // ======================= TMA producer =======================
      // Physical pages of K/V tile j (paged): the table entries are read
      // together, once per tile, for both the K and the V copies.  Pages past
      // the sequence, and entries outside the pool (flagged), read page 0: the
      // pool's contents are finite and those keys are masked.
      constexpr int kMaxPagesPerTile = kBN / 8;
      int phys[kMaxPagesPerTile];
      auto lookup_pages = [&](const Item& it, int j) {
        if constexpr (kPaged) {
          const int per_tile = kBN / a.page_size;
          const int32_t* row = a.block_table + static_cast<size_t>(it.b) * a.max_pages + j * per_tile;
#pragma unroll
          for (int p = 0; p < kMaxPagesPerTile; ++p)
            phys[p] = (p < per_tile && (j * per_tile + p) * a.page_size < it.Nkv) ? __ldg(row + p) : 0;
#pragma unroll
          for (int p = 0; p < kMaxPagesPerTile; ++p)
            if (phys[p] < 0 || phys[p] >= a.num_pages_total) {
              atomicOr(a.status, kDevBadBlockTable);
              phys[p] = 0;
            }
        }
      };
      // K or V tile j into ring slot `dst`: one tile box (dense), or one box per
      // page (paged, pages from lookup_pages).  With two 64-column chunks a page
      // arrives in one copy, not one per chunk: a copy's fixed cost, not its
      // bytes, is what a small page pays for.  Paged V is page-major
      // ([page][chunk][page rows][128 B]): each 16-key step of P V addresses its
      // own page block.  Paged K uses the 32-byte swizzle as
      // [8-row group][16-column K step][8 rows][32 B]: the scores MMA reads each
      // K step of all 128 keys at one 8-row-group stride (2 KB), whichever page
      // the group came from.
      auto load_kv = [&](const Item& it, const CUtensorMap* tm, uint32_t dst, uint32_t bar, int j, bool is_v) {
        if constexpr (kPaged) {
          const int per_tile = kBN / a.page_size;
#pragma unroll
          for (int p = 0; p < kMaxPagesPerTile; ++p) {
            if (p >= per_tile) break;
            if (L::kChunks == 2 && is_v) {
              tma_load_5d(dst + p * a.page_size * 256, tm, bar, 0, 0, 0, it.hkv, phys[p]);
            } else if (L::kChunks == 2) {
              tma_load_5d(dst + p * a.page_size * 256, tm, bar, 0, 0, 0, 0, phys[p] * a.Hkv + it.hkv);
            } else {
              for (int c = 0; c < L::kChunks; ++c)
                tma_load_4d(dst + c * L::kChunkBytes + p * a.page_size * 128, tm, bar, c * L::kChunkElems, 0,
                            it.hkv, phys[p]);
            }
          }
        } else {
          tma_load_4d(dst, tm, bar, 0, j * kBN, 0, it.b * a.Hkv + it.hkv);
        }
      };
      bool ok = true;
      uint32_t g = 0;            // K/V tiles loaded so far: ring slot g % S, use (g / S)
      uint32_t gk = 0, gv = 0;   // K and V copies issued (for the drain)
      int qi = 0;                // items whose Q tiles were loaded
      int requested = 0;         // work requests made (the last one's answer is awaited before exit)
      int answered = 0;
      int idx = static_cast<int>(blockIdx.x);
      for (int k = 0; idx >= 0 && ok; ++k) {
        // ask for the item after this one now, so the answer is back by the time it is needed
        if constexpr (kPersistent) {
          const int kn = k + 1, sl = kn & 1;
          if (kn >= 3 && !(ok = mbar_wait(BAR_ITE(sl), resp_parity(kn - 2), a.status, abort_flag))) break;
          fence_proxy_async_smem();   // the slot's previous answer was read through the generic proxy
          mbar_arrive_expect_tx(BAR_ITF(sl), 16);
          clc_try_cancel(sResp + 16 * sl, BAR_ITF(sl));
          requested = kn;
        }
        const Item it = decode_item(idx, true);
        if (it.valid) {
          // this buffer's previous Q tiles are free once the last Q.K^T reading them completed
          if (qi > 0 && !(ok = mbar_wait(BAR_QE(), static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag)))
            break;
          const uint32_t qbytes = static_cast<uint32_t>((it.q0_0 < it.Nq) + (it.q0_1 < it.Nq)) * L::kTileBytes;
          mbar_arrive_expect_tx(BAR_Q(), qbytes);
          for (int t = 0; t < 2; ++t) {
            const int q0 = t ? it.q0_1 : it.q0_0;
            const int hq = t ? it.hq_1 : it.hq_0;
            if (q0 >= it.Nq) continue;
            if constexpr (kPaged)   // packed [total_q, Hq, d]: box of 128 rows of one head
              tma_load_4d(sQ + t * L::kTileBytes, &tmQ, BAR_Q(), 0, hq, it.q_base + q0, 0);
            else
              tma_load_4d(sQ + t * L::kTileBytes, &tmQ, BAR_Q(), 0, q0, 0, it.b * a.Hq + hq);
          }
          ++qi;
          for (int j = 0; j < it.n_max && ok; ++j, ++g) {
            const int s = static_cast<int>(g % L::kStages);
            const uint32_t ph = (g / L::kStages) & 1u;
            lookup_pages(it, j);   // before the wait, so the table reads overlap it
            if (!(ok = mbar_wait(BAR_KE(s), ph ^ 1u, a.status, abort_flag))) break;
            mbar_arrive_expect_tx(BAR_KF(s), L::kTileBytes);
            load_kv(it, &tmK, sK + s * L::kTileBytes, BAR_KF(s), j, false);
            ++gk;
            if (!(ok = mbar_wait(BAR_VE(s), ph ^ 1u, a.status, abort_flag))) break;
            mbar_arrive_expect_tx(BAR_VF(s), L::kTileBytes);
            load_kv(it, &tmV, sV + s * L::kTileBytes, BAR_VF(s), j, true);
            ++gv;
          }
          if (!ok) break;
        }
        // the next item (or none)
        if constexpr (!kPersistent) break;
        const int kn = k + 1, sl = kn & 1;
        if (!(ok = mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
        answered = kn;
        idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      }
      // drain: no copy into this CTA's shared memory may still be in flight at exit
      if (answered < requested)
        mbar_wait(BAR_ITF(requested & 1), resp_parity(requested), nullptr, nullptr, kWaitLimitNs);
      if (qi > 0) mbar_wait(BAR_Q(), static_cast<uint32_t>(qi - 1) & 1u, nullptr, nullptr, kWaitLimitNs);
      constexpr uint32_t kS = L::kStages;
      for (uint32_t gg = (gk > kS ? gk - kS : 0u); gg < gk; ++gg)
        mbar_wait(BAR_KF(static_cast<int>(gg % kS)), (gg / kS) & 1u, nullptr, nullptr, kWaitLimitNs);
      for (uint32_t gg = (gv > kS ? gv - kS : 0u); gg < gv; ++gg)
        mbar_wait(BAR_VF(static_cast<int>(gg % kS)), (gg / kS) & 1u, nullptr, nullptr, kWaitLimitNs);
    } else if (warp == 1) {
    // ======================= MMA issuer =======================
      // The whole warp runs the issue loop (warp-uniform descriptors and
      // waits); the elected lane issues the MMAs and their commits.
      const bool leader = elect_one_sync();
      constexpr uint32_t idesc_qk = kFp8 ? idesc_e4m3_f32(kBM, kBN, false) : idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = kFp8 ? idesc_e4m3_f32(kBM, D, true) : idesc_bf16_f32(kBM, D, true);
      // The leader issues a whole product inside one branch: a branch around
      // every MMA made issue about as slow as the tensor pipe's execution of
      // a 128 x 128 x 16 step.
      auto mma_s = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
        if constexpr (kFp8) mma_ss_f8(d, ad, bd, id, acc); else mma_ss(d, ad, bd, id, acc);
      };
      auto mma_t = [&](uint32_t d, uint32_t at, uint64_t bd, uint32_t id, uint32_t acc) {
        if constexpr (kFp8) mma_ts_f8(d, at, bd, id, acc); else mma_ts(d, at, bd, id, acc);
      };
      // commits come from the lane that issued the MMAs they cover
      auto commit = [&](uint32_t bar) {
        if (leader) mma_commit(bar);
        __syncwarp();
      };
      auto tS = [&](int t) { return tmem + (t ? L::kTmS1 : L::kTmS0); };
      auto tO = [&](int t) { return tmem + (t ? L::kTmO1 : L::kTmO0); };

      // Shared-memory descriptors are built once; a K step or a ring stage
      // only moves the start-address field (address >> 4), so the issue loop
      // adds compile-time offsets instead of rebuilding descriptors.
      const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
      // paged K with two chunks: 32-byte swizzle, K step kk at byte 256 kk
      constexpr bool kPagedK = kPaged && L::kChunks == 2;
      const uint64_t dK = kPagedK ? smem_desc_sw32(sK, 2048) : smem_desc_sw128(sK, 16, 1024);
      constexpr uint64_t kKStep = kPagedK ? 16 : 2;                              // one K step
      constexpr uint64_t kKChunk = kPagedK ? 4 * kKStep : (L::kChunkBytes >> 4);   // four K steps
      // Paged V with two chunks is page-major: the chunk stride is one page of
      // 128-byte rows; 8-key groups are 1024 bytes apart inside a page, one
      // page block (2 KB) apart when a page holds 8 keys.
      constexpr bool kPagedV = kPaged && L::kChunks == 2;
      const int ps = kPaged ? a.page_size : 128;
      const uint64_t dV = kPagedV ? smem_desc_sw128(sV, static_cast<uint32_t>(ps) * 128u, ps >= 16 ? 1024u : 2048u)
                                  : smem_desc_sw128(sV, L::kChunkBytes, 1024);
      constexpr uint64_t kTileStep = L::kTileBytes >> 4;
      // 16-key step kk starts at byte 2048 (kk + (kk & vmask)): m = max(page / 16, 1) steps per
      // page (a power of two), page blocks of m * 4096 bytes, 2048 bytes per step inside one
      const int vmask = ~(max(ps / 16, 1) - 1);

      // S_t = Q_t K^T over d in 32-byte steps (K-major operands, 128B swizzle)
      auto issue_qk = [&](int t, int s) {
        uint64_t a0 = dQ + static_cast<uint64_t>(t) * kTileStep;
        uint64_t b0 = dK + static_cast<uint64_t>(s) * kTileStep;
        const uint32_t d = tS(t);
        // K steps of 32 bytes (16 bf16 or 32 fp8 elements) within a 128-byte
        // swizzle row, then the next 128-byte chunk of d
        if (leader) {
#pragma unroll 1
          for (int c = 0; c < L::kChunks; ++c) {
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              mma_s(d, a0 + 2 * k4, b0 + kKStep * k4, idesc_qk, (c | k4) != 0 ? 1u : 0u);
            a0 += L::kChunkBytes >> 4;
            b0 += kKChunk;
          }
        }
        __syncwarp();
      };
      // O_t += P_t V over one half (64 keys) of the tile, 16 (bf16) or 32
      // (fp8) keys per MMA (P from TMEM: 8 columns per step either way; V
      // MN-major, one 128-byte row per key)
      auto issue_pv_half = [&](int t, int s, int half, bool acc) {
        constexpr int kPerHalf = (kBN / 2) / L::kKeysPerMma;
        const uint64_t b0 = dV + static_cast<uint64_t>(s) * kTileStep;
        const uint32_t d = tO(t), a = tS(t);
        if (leader) {
#pragma unroll
          for (int k4 = 0; k4 < kPerHalf; ++k4) {
            const int kk = half * kPerHalf + k4;
            uint32_t off = kk * L::kKeysPerMma * 128;   // dense: 16 keys of 128-byte rows per step
            if constexpr (kPagedV) {
              off = static_cast<uint32_t>((kk + (kk & vmask)) << 11);
            }
            mma_t(d, a + kk * 8, b0 + static_cast<uint64_t>(off >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };

      bool ok = true;
      uint32_t g = 0;              // K/V tiles consumed (ring position, as the producer's)
      uint32_t steps[2] = {0, 0};  // K/V steps of each query tile so far: S/P/O barrier phases
      int qi = 0;                  // items whose Q tiles were used
      int idx = static_cast<int>(blockIdx.x);
      for (int k = 0; idx >= 0 && ok; ++k) {
        const Item it = decode_item(idx, false);
        if (it.valid) {
          if (!(ok = mbar_wait_warp(BAR_Q(), static_cast<uint32_t>(qi) & 1u, a.status, abort_flag))) break;
          tc_fence_after();
          if (it.n_max > 0) {
            const int s0 = static_cast<int>(g % L::kStages);
            if (!(ok = mbar_wait_warp(BAR_KF(s0), (g / L::kStages) & 1u, a.status, abort_flag))) break;
            tc_fence_after();
            for (int t = 0; t < 2; ++t)
              if ((t ? it.nt_1 : it.nt_0) > 0) {
                issue_qk(t, s0);
                commit(BAR_SF(t));
              }
            commit(BAR_KE(s0));
          }
          if (it.n_max <= 1) commit(BAR_QE());   // no later Q.K^T of this item reads Q
          for (int j = 0; j < it.n_max && ok; ++j) {
            const uint32_t gj = g + static_cast<uint32_t>(j);
            const int s = static_cast<int>(gj % L::kStages);
            const uint32_t ph = (gj / L::kStages) & 1u;
            const int s1 = static_cast<int>((gj + 1) % L::kStages);
            const uint32_t ph1 = ((gj + 1) / L::kStages) & 1u;
            if (!(ok = mbar_wait_warp(BAR_VF(s), ph, a.status, abort_flag))) break;
            for (int t = 0; t < 2; ++t) {
              const int ntt = t ? it.nt_1 : it.nt_0;
              if (j >= ntt) continue;
              const uint32_t c = steps[t];
              // the first P.V of an item overwrites O_t: the previous item's
              // epilogue must have read it
              if (j == 0 && qi > 0 &&
                  !(ok = mbar_wait_warp(BAR_OF(t), static_cast<uint32_t>(qi - 1) & 1u, a.status, abort_flag)))
                break;
              if (!(ok = mbar_wait_warp(BAR_PH(t), c & 1u, a.status, abort_flag))) break;
              tc_fence_after();
              issue_pv_half(t, s, 0, j > 0);
              if (!(ok = mbar_wait_warp(BAR_PR(t), c & 1u, a.status, abort_flag))) break;
              tc_fence_after();
              issue_pv_half(t, s, 1, true);
              commit(BAR_OD(t));
              if (j + 1 < ntt) {
                if (!(ok = mbar_wait_warp(BAR_KF(s1), ph1, a.status, abort_flag))) break;
                issue_qk(t, s1);
                commit(BAR_SF(t));
              }
              steps[t] = c + 1;
            }
            if (!ok) break;
            if (j + 2 == it.n_max) commit(BAR_QE());   // the item's last Q.K^T has been issued
            commit(BAR_VE(s));
            if (j + 1 < it.n_max) commit(BAR_KE(s1));
          }
          if (!ok) break;
          g += static_cast<uint32_t>(it.n_max);
          ++qi;
        }
        // the next item (or none)
        if constexpr (!kPersistent) break;
        const int kn = k + 1, sl = kn & 1;
        if (!(ok = mbar_wait_warp(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag))) break;
        idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
        __syncwarp();
        if (leader) mbar_arrive(BAR_ITE(sl));
      }
      // no commit may still be pending when the CTA exits
      commit(BAR_FIN());
      mbar_wait_warp(BAR_FIN(), 0, nullptr, nullptr);
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ======================= softmax warpgroups =======================
    const int t = (warp - kSoftmaxWarp0) / 4;           // query tile of this warpgroup
    const int quarter = warp & 3;                       // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;                // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + (t == 0 ? L::kTmS0 : L::kTmS1) + lane_off;
    const uint32_t tO = tmem + (t == 0 ? L::kTmO0 : L::kTmO1) + lane_off;
    const float c2 = a.scale_log2;
    bool ok = true;
    uint32_t steps = 0;    // K/V steps of this tile so far: S/P/O barrier phases
    int idx = static_cast<int>(blockIdx.x);
    for (int k = 0; idx >= 0 && ok; ++k) {
      const Item it = decode_item(idx, false);
      if (it.valid) {
        const int q0 = t ? it.q0_1 : it.q0_0;               // first query row of the tile
        const int hq = t ? it.hq_1 : it.hq_0;               // query head of the tile
        const int qrow = q0 + row;                          // query index
        const int Nq = it.Nq, Nkv = it.Nkv;
        const int n = t ? it.nt_1 : it.nt_0;
        const int off = Nkv - Nq;
        // visible keys of this row: [0, vis_end)
        const int vis_end = a.causal ? min(Nkv, qrow + off + 1) : Nkv;

        float m = -INFINITY;  // running max of the raw scores q.k
        float l = 0.f;        // running sum of exp2((s - m) * c2)

        for (int j = 0; j < n; ++j) {
          ok = mbar_wait(BAR_SF(t), (steps + j) & 1u, a.status, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          uint32_t sr[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
          tmem_wait_ld();
          float* s = reinterpret_cast<float*>(&sr[0][0]);

          // tile-uniform: does any row of this tile have masked keys in tile j?
          const int kv0 = j * kBN;
          const bool need_mask =
              (kv0 + kBN > Nkv) || (a.causal && kv0 + kBN - 1 > q0 + off);
          const int lim = vis_end - kv0;  // visible columns of this tile for this row: [0, lim)
          if (need_mask) {
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = c < lim ? s[c] : -INFINITY;
          }

          // exp2((s - m) * c2) for 32 column pairs [64h, 64h + 64), packed to bf16
          // pairs (32 words) or to four E4M3 codes per word (fp8: 16 words);
          // masked columns get exactly 0.  Returns the sum of the unrounded values.
          // The masked form is a separate specialisation so unmasked tiles carry
          // no per-element compare/select.
          auto exp_half = [&](auto masked, int h, float negm, uint32_t (&pk)[L::kPWords]) -> float {
            constexpr bool kMasked = decltype(masked)::value;
            const float2 c2v = make_float2(c2, c2), negv = make_float2(negm, negm);
            float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
            float2 pp_prev = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = h * 64 + 2 * i;
              const float2 x = ffma2(make_float2(s[c], s[c + 1]), c2v, negv);
              float2 pp;
              if (((kFp8 ? kPolyMaskFp8 : kPolyMask) >> (i & 7)) & 1u) {
                pp = exp2_poly2(x);
              } else {
                pp.x = ex2(x.x);
                pp.y = ex2(x.y);
              }
              if constexpr (kMasked) {
                pp.x = c < lim ? pp.x : 0.f;
                pp.y = c + 1 < lim ? pp.y : 0.f;
              }
              if (i & 1) {
                sb = fadd2(sb, pp);
              } else {
                sa = fadd2(sa, pp);
              }
              if constexpr (kFp8) {
                if (i & 1) pk[i >> 1] = pack_e4m3x4(pp_prev.x, pp_prev.y, pp.x, pp.y);
                pp_prev = pp;
              } else {
                pk[i] = pack_bf16x2(pp.x, pp.y);
              }
            }
            return (sa.x + sb.x) + (sa.y + sb.y);
          };
          auto exp_half_any = [&](int h, float negm, uint32_t (&pk)[L::kPWords]) -> float {
            return need_mask ? exp_half(std::true_type{}, h, negm, pk) : exp_half(std::false_type{}, h, negm, pk);
          };

          // row max of the tile, then the running max with a stale-max margin:
          // the max is only moved (and O rescaled) when it grows by more than
          // 2^8 in exp2 units; weights stay below 2^8 either way.
          float mx;
          {
            float r0 = -INFINITY, r1 = -INFINITY, r2 = -INFINITY, r3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
              r0 = fmax3(r0, s[c + 0], s[c + 1]);
              r1 = fmax3(r1, s[c + 2], s[c + 3]);
              r2 = fmax3(r2, s[c + 4], s[c + 5]);
              r3 = fmax3(r3, s[c + 6], s[c + 7]);
            }
            mx = fmaxf(fmax3(r0, r1, r2), r3);
          }
          const float m_new = fmaxf(m, mx);
          const bool upd = (m == -INFINITY) || ((m_new - m) * c2 > kRescaleLog2);
          const float m_use = upd ? m_new : m;
          const float alpha = (upd && m != -INFINITY) ? ex2((m - m_use) * c2) : (m == -INFINITY ? 0.f : 1.f);
          const float negm = (m_use == -INFINITY) ? 0.f : -m_use * c2;
          m = m_use;

          // Rescale O before any of this tile's P.V lands on it.  The previous
          // P.V has completed: the commit that signalled this S tile was issued
          // after it and covers every earlier MMA.
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(tO + c * 32, orr);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(tO + c * 32, orr);
            }
          }

          // P (bf16 pairs) into the first 64 columns of this tile's S region, one
          // half (64 keys) at a time; the MMA warp starts P.V on the first half
          // while the second is computed.
          float psum;
          {
            uint32_t pk[L::kPWords];
            psum = exp_half_any(0, negm, pk);
            if constexpr (kFp8) tmem_st16(tS, pk); else tmem_st32(tS, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(BAR_PH(t));
          {
            uint32_t pk[L::kPWords];
            psum += exp_half_any(1, negm, pk);
            if constexpr (kFp8) tmem_st16(tS + L::kPWords, pk); else tmem_st32(tS + L::kPWords, pk);
          }
          l = alpha * l + psum;

          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(BAR_PR(t));
        }

        // ---- epilogue: O / l -> bf16, lse = m * scale + ln(l)
        const bool have = (n > 0) && ok;
        if (have) {
          ok = mbar_wait(BAR_OD(t), (steps + n - 1) & 1u, a.status, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          tc_fence_after();
        }
        steps += static_cast<uint32_t>(n);
        const bool store = qrow < Nq;
        // output row: [B, Hq, Nq] (dense) or packed [total_q, Hq] (paged).  O
        // leaves by 16-byte stores per thread: the Q buffer may already hold the
        // next item's tiles.
        const size_t orow = kPaged ? static_cast<size_t>(it.q_base + (store ? qrow : 0)) * a.Hq + hq
                                   : (static_cast<size_t>(it.b) * a.Hq + hq) * Nq + qrow;
        const float inv = (l > 0.f) ? (kFp8 ? a.v_descale / l : 1.f / l) : 0.f;
        __nv_bfloat16* optr = a.o + orow * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          if (have && ok) {
            tmem_ld32(tO + c * 32, orr);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = 0u;
          }
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(optr + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(orr[8 * e + 0]) * inv, __uint_as_float(orr[8 * e + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(orr[8 * e + 2]) * inv, __uint_as_float(orr[8 * e + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(orr[8 * e + 4]) * inv, __uint_as_float(orr[8 * e + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(orr[8 * e + 6]) * inv, __uint_as_float(orr[8 * e + 7]) * inv);
              dst[e] = w;
            }
          }
        }
        // O_t has been read: the next item's first P.V may overwrite it
        tc_fence_before();
        mbar_arrive(BAR_OF(t));
        if (store && a.lse) {
          a.lse[orow] = (l > 0.f) ? fmaf(m, a.scale, __log2f(l) * 0.69314718055994531f) : -INFINITY;
        }
      }   // valid item
      // the next item (or none)
      if constexpr (!kPersistent) break;
      const int kn = k + 1, sl = kn & 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(BAR_ITF(sl), resp_parity(kn), a.status, abort_flag));
      if (!ok) break;
      idx = clc_cancelled_ctaid_x(sResp + 16 * sl);
      mbar_arrive(BAR_ITE(sl));
    }   // items
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Work units: with an even number of query heads per KV head, a CTA takes one
// 128-row tile of two heads of a group (equal work for both softmax
// warpgroups, no half-empty last pair); otherwise two consecutive tiles of one
// head.  max_q is Nq (dense) or the longest query chunk (paged).
static void set_units(PrefillArgs& a, int Hq, int Hkv, int max_q) {
  a.head_pair = ((Hq / Hkv) % 2 == 0) ? 1 : 0;
  a.n_units = a.head_pair ? (max_q + kBM - 1) / kBM : (max_q + 2 * kBM - 1) / (2 * kBM);
}

// Output for shapes with no keys at all: O = 0, lse = -inf.
__global__ void empty_keys_kernel(__nv_bfloat16* o, float* lse, size_t rows, int d) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i < rows * d) o[i] = __float2bfloat16(0.f);
  if (lse && i < rows) lse[i] = -INFINITY;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int D>
static ta_status launch_prefill_d(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                  int Hkv, int Nq, int Nkv, float scale, int causal, cudaStream_t stream) {
  using L = PrefillLayout<D>;
  CUtensorMap tq, tk, tv;
  ta_status st;
  if ((st = encode_rows_chunked(&tq, q, D, Nq, B * Hq)) != TA_OK) return st;
  if ((st = encode_rows_chunked(&tk, k, D, Nkv, B * Hkv)) != TA_OK) return st;
  if ((st = encode_rows_chunked(&tv, v, D, Nkv, B * Hkv)) != TA_OK) return st;
  static int attr_done[64] = {0};
  cudaError_t e = ensure_smem_limit(prefill_fwd_kernel<D, false, false>, L::kAlloc, attr_done);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "prefill: shared-memory limit", e);
  PrefillArgs a = {};
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  set_units(a, Hq, Hkv, Nq);
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.v_descale = 1.f;
  a.status = device_status_ptr();
  if (!a.status) return fail(TA_ERR_CUDA, "prefill: device status word");
  const unsigned grid = static_cast<unsigned>(a.n_units) * static_cast<unsigned>(B * Hq / (a.head_pair + 1));
  prefill_fwd_kernel<D, false, false><<<grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, a);
  e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "prefill: launch", e);
}

template <int D>
static ta_status launch_paged_prefill_d(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_table, const int32_t* cu_seqlens,
                                        const int32_t* seq_lens, int page_size, int num_seqs, int total_q,
                                        int max_q_len, int Hq, int Hkv, int max_pages, int num_pages_total,
                                        float scale, int causal, void* o, float* lse, cudaStream_t stream) {
  using L = PrefillLayout<D>;
  CUtensorMap tq, tk, tv;
  ta_status st;
  {  // packed queries [total_q, Hq, d] as {64, Hq, total_q, d / 64}: one box of 128 rows of one head
     // lands as [chunk][128 rows][128 B]
    const uint64_t dims[4] = {64, static_cast<uint64_t>(Hq), static_cast<uint64_t>(total_q), D / 64};
    const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hq) * D * 2, 128};
    const uint32_t box[4] = {64, 1, 128, D / 64};
    if ((st = encode_bf16_tiled(&tq, q, 4, dims, strides, box)) != TA_OK) return st;
  }
  {  // pool [P, Hkv, page, d]: boxes of one page of one KV head
    const uint64_t dims[4] = {D, static_cast<uint64_t>(page_size), static_cast<uint64_t>(Hkv),
                              static_cast<uint64_t>(num_pages_total)};
    const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(page_size) * D * 2,
                                 static_cast<uint64_t>(Hkv) * page_size * D * 2};
    const uint32_t box[4] = {64, static_cast<uint32_t>(page_size), 1, 1};
    if (L::kChunks == 1) {
      if ((st = encode_bf16_tiled(&tk, k_cache, 4, dims, strides, box)) != TA_OK) return st;
      if ((st = encode_bf16_tiled(&tv, v_cache, 4, dims, strides, box)) != TA_OK) return st;
    } else {
      // K: [P, Hkv, page, 128] seen as 5-D {16 columns, 8 rows, 8 column groups, page / 8 row
      // groups, P * Hkv (page, head) blocks}, box {16, 8, 8, page / 8, 1}, 32-byte swizzle: one
      // copy lands a page as [row group][column group][8 rows][32 B]
      const uint64_t dk[5] = {16, 8, 8, static_cast<uint64_t>(page_size / 8),
                              static_cast<uint64_t>(num_pages_total) * Hkv};
      const uint64_t sk[4] = {static_cast<uint64_t>(D) * 2, 32, 8ull * D * 2, static_cast<uint64_t>(page_size) * D * 2};
      const uint32_t bk[5] = {16, 8, 8, static_cast<uint32_t>(page_size / 8), 1};
      if ((st = encode_bf16_tiled_sw32(&tk, k_cache, 5, dk, sk, bk)) != TA_OK) return st;
      // V: [P, Hkv, page, (2 chunks of 64)] seen as 5-D {64, page, chunk, Hkv, P}, so that one box
      // {64, page, 2, 1, 1} lands a page as [chunk][page rows][128 B]
      const uint64_t dv[5] = {64, static_cast<uint64_t>(page_size), 2, static_cast<uint64_t>(Hkv),
                              static_cast<uint64_t>(num_pages_total)};
      const uint64_t sv[4] = {static_cast<uint64_t>(D) * 2, 128, static_cast<uint64_t>(page_size) * D * 2,
                              static_cast<uint64_t>(Hkv) * page_size * D * 2};
      const uint32_t bv[5] = {64, static_cast<uint32_t>(page_size), 2, 1, 1};
      if ((st = encode_bf16_tiled(&tv, v_cache, 5, dv, sv, bv)) != TA_OK) return st;
    }
  }
  static int attr_done[64] = {0};
  cudaError_t e = ensure_smem_limit(prefill_fwd_kernel<D, true, false>, L::kAlloc, attr_done);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "paged prefill: shared-memory limit", e);
  PrefillArgs a = {};
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.B = 1;
  a.Hq = Hq;
  a.Hkv = Hkv;
  set_units(a, Hq, Hkv, max_q_len);
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.v_descale = 1.f;
  a.status = device_status_ptr();
  if (!a.status) return fail(TA_ERR_CUDA, "paged prefill: device status word");
  a.block_table = block_table;
  a.cu_seqlens = cu_seqlens;
  a.seq_lens = seq_lens;
  a.num_seqs = num_seqs;
  a.total_q = total_q;
  a.max_q_len = max_q_len;
  a.page_size = page_size;
  a.max_pages = max_pages;
  a.num_pages_total = num_pages_total;
  const unsigned grid = static_cast<unsigned>(a.n_units) * static_cast<unsigned>(num_seqs * Hq / (a.head_pair + 1));
  prefill_fwd_kernel<D, true, false><<<grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, a);
  e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "paged prefill: launch", e);
}

// FP8 (E4M3) inputs, d = 128: Q, K, V [B, H, N, 128] one byte per element.
// The descales of q and k multiply every score, so they join the softmax
// scale; v's multiplies O.
ta_status launch_prefill_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale,
                             float v_descale, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nkv,
                             float scale, int causal, cudaStream_t stream) {
  constexpr int D = 128;
  using L = PrefillLayout<D, true>;
  if (B == 0 || Nq == 0) return TA_OK;
  if (Nkv == 0) {
    const size_t rows = static_cast<size_t>(B) * Hq * Nq;
    const size_t n = rows * D;
    empty_keys_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        static_cast<__nv_bfloat16*>(o), lse, rows, D);
    return cudaGetLastError() == cudaSuccess ? TA_OK : TA_ERR_CUDA;
  }
  CUtensorMap tq, tk, tv;
  ta_status st;
  if ((st = encode_u8_rows_chunked(&tq, q, D, Nq, B * Hq)) != TA_OK) return st;
  if ((st = encode_u8_rows_chunked(&tk, k, D, Nkv, B * Hkv)) != TA_OK) return st;
  if ((st = encode_u8_rows_chunked(&tv, v, D, Nkv, B * Hkv)) != TA_OK) return st;
  static int attr_done[64] = {0};
  cudaError_t e = ensure_smem_limit(prefill_fwd_kernel<D, false, true>, L::kAlloc, attr_done);
  if (e != cudaSuccess) return fail(TA_ERR_CUDA, "fp8 prefill: shared-memory limit", e);
  const float s = scale * q_descale * k_descale;
  PrefillArgs a = {};
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  set_units(a, Hq, Hkv, Nq);
  a.causal = causal;
  a.scale = s;
  a.scale_log2 = s * 1.4426950408889634f;
  a.v_descale = v_descale;
  a.status = device_status_ptr();
  if (!a.status) return fail(TA_ERR_CUDA, "fp8 prefill: device status word");
  const unsigned grid = static_cast<unsigned>(a.n_units) * static_cast<unsigned>(B * Hq / (a.head_pair + 1));
  prefill_fwd_kernel<D, false, true><<<grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, a);
  e = cudaGetLastError();
  return e == cudaSuccess ? TA_OK : fail(TA_ERR_CUDA, "fp8 prefill: launch", e);
}

ta_status launch_paged_prefill(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                               const int32_t* cu_seqlens, const int32_t* seq_lens, int page_size, int num_seqs,
                               int total_q, int max_q_len, int Hq, int Hkv, int d, int max_pages,
                               int num_pages_total, float scale, int causal, void* o, float* lse,
                               cudaStream_t stream) {
  if (d == 128)
    return launch_paged_prefill_d<128>(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, page_size, num_seqs,
                                       total_q, max_q_len, Hq, Hkv, max_pages, num_pages_total, scale, causal, o,
                                       lse, stream);
  return launch_paged_prefill_d<64>(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, page_size, num_seqs,
                                    total_q, max_q_len, Hq, Hkv, max_pages, num_pages_total, scale, causal, o, lse,
                                    stream);
}

ta_status launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                         int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  if (B == 0 || Nq == 0) return TA_OK;
  if (Nkv == 0) {
    const size_t rows = static_cast<size_t>(B) * Hq * Nq;
    const size_t n = rows * d;
    empty_keys_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        static_cast<__nv_bfloat16*>(o), lse, rows, d);
    return cudaGetLastError() == cudaSuccess ? TA_OK : TA_ERR_CUDA;
  }
  if (d == 128) return launch_prefill_d<128>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
  return launch_prefill_d<64>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
}

}  // namespace ta
