/*
 * tiledattn.h - C ABI of the B200 fused tiled-attention library (libtiledattn.so).
 *
 * The library computes exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 *
 * in one fused, tiled pass (online softmax: running row max m and sum l,
 * rescaling of the partial output on every new K/V tile), so the N x N score
 * and probability matrices never reach HBM.  Problem statement: Gemini 3 Flash
 * kernel-fusion post, sections "traditional attention" (S = QK^T, P = softmax(S),
 * O = PV) and 1-3 (fusion, tiling, online softmax); FlashAttention optimisation
 * article, sections 2.1 and 3.1-3.2.
 *
 * Conventions shared by every call
 *  - All Q/K/V/O arrays are bfloat16 (attn_fwd_fp8: Q/K/V as E4M3 codes),
 *    dense, row-major, with 16-byte aligned base pointers (128-byte alignment
 *    recommended; FlashAttention article 5.2, kernel-fusion post "data
 *    layout").  lse arrays are float32.
 *  - Pointers are DEVICE pointers unless stated otherwise.  The caller owns
 *    every buffer and the stream.  No call allocates memory or synchronises;
 *    work is enqueued on `stream` and the call returns.
 *  - Argument errors are detected on the host before anything is enqueued and
 *    return TA_ERR_INVALID_ARG or TA_ERR_UNSUPPORTED.  A failed launch returns
 *    TA_ERR_CUDA.  Faults found on the device (a block-table entry outside the
 *    pool, a bounded wait that gave up) never trap: the kernel clamps or skips,
 *    records a bit in a device status word, and the caller may read that word
 *    with attn_paged_decode_check() / ta_device_status().
 *  - Grouped-query attention: query head hq reads KV head hq / (Hq / Hkv), i.e.
 *    consecutive query heads share a KV head (GPU-optimisation tag page, GQA).
 *  - Causal masking is aligned to the bottom-right corner: query i sees keys
 *    j <= i + (Nkv - Nq).  A query with no visible key gets O = 0, lse = -inf.
 *  - lse (optional, may be NULL) is the natural log of the softmax normaliser
 *    of the scaled scores: lse = m + ln(sum_j exp(s_j - m)).  It is the per-row
 *    max and normaliser the kernel-fusion post (section 4) keeps for a
 *    recomputing backward pass.
 */
#ifndef TILEDATTN_H
#define TILEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without requiring the CUDA headers; NULL = legacy default stream. */
typedef struct CUstream_st *ta_stream_t;

typedef enum {
    TA_OK = 0,
    TA_ERR_INVALID_ARG = 1,     /* bad pointer, shape, alignment or size */
    TA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (head dim, page size, ...) */
    TA_ERR_CUDA = 3,            /* a CUDA runtime/driver call failed */
    TA_ERR_BAD_BLOCK_TABLE = 4, /* a block-table entry or length was out of range */
    TA_ERR_DEVICE_TIMEOUT = 5   /* a bounded device-side wait gave up */
} ta_status;

/* Bits of the device status word. */
#define TA_DEV_TIMEOUT 1u
#define TA_DEV_BAD_BLOCK_TABLE 2u
#define TA_DEV_BAD_SEQ_LEN 4u

/* Human-readable name of a status code (static string, never NULL). */
const char *ta_status_string(ta_status status);

/* Library version as major*10000 + minor*100 + patch. */
int ta_version(void);

/*
 * Description of the last host-side failure on the calling thread (which step
 * failed and the CUDA error name), or "" if none.  Static thread-local
 * storage, never NULL; overwritten by the next failure.
 */
const char *ta_last_error(void);

/*
 * attn_fwd - fused attention forward (prefill).
 *
 *   q   [B, Hq,  Nq,  d]  bf16     o   [B, Hq, Nq, d] bf16 (written)
 *   k   [B, Hkv, Nkv, d]  bf16     lse [B, Hq, Nq]    fp32 (written; may be NULL)
 *   v   [B, Hkv, Nkv, d]  bf16
 *
 * scale: multiplier of the scores (1/sqrt(d) in the pages' statement,
 * GPU-optimisation tag page "algorithm principle"); must be finite and >= 0.
 * causal: 0 or 1.  Supported: d in {64, 128}, Hq % Hkv == 0, all sizes >= 0
 * (B*Hq*Nq == 0 does nothing; Nkv == 0 writes O = 0, lse = -inf).
 * o must not overlap q, k or v.
 */
ta_status attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                   float scale, int causal, ta_stream_t stream);

/*
 * attn_fwd_fp8 - fused attention forward with FP8 inputs (the FP8 tensor-core
 * variant of the LLM-inference page's Flash Attention V3 section).
 *
 *   q   [B, Hq,  Nq,  d]  E4M3 codes  o   [B, Hq, Nq, d] bf16 (written)
 *   k   [B, Hkv, Nkv, d]  E4M3 codes  lse [B, Hq, Nq]    fp32 (written; may be NULL)
 *   v   [B, Hkv, Nkv, d]  E4M3 codes
 *
 * One byte per element in the OCP E4M3 form ("e4m3fn": bias 7, no infinity,
 * largest finite 448).  The real inputs are q_descale * e4m3(q), k_descale *
 * e4m3(k), v_descale * e4m3(v) (one factor per tensor, finite and > 0), and
 * the result approximates the attention of those values: the scores are
 * exact products accumulated in fp32, but the softmax weights are rounded to
 * E4M3 for the FP8 P.V product (relative error up to 2^-4 per weight, about
 * 2.6% RMS), so O carries an error of a few percent of its magnitude; lse is
 * as accurate as attn_fwd's.  Scale, causal alignment, GQA mapping, empty
 * cases and alignment rules as attn_fwd.  Supported: d = 128.
 */
ta_status attn_fwd_fp8(const void *q, const void *k, const void *v, float q_descale, float k_descale,
                       float v_descale, void *o, float *lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                       float scale, int causal, ta_stream_t stream);

/*
 * attn_paged_prefill - varlen (chunked) prefill against the paged KV cache:
 * the new query tokens of several sequences, packed, attend over their
 * sequences' keys in the page pool (chunked prefill, LLM-inference article
 * section 3.2; PagedAttention, GPU-optimisation tag page; block gather,
 * paged-gather article section 2).  The new tokens' K/V must already be in
 * the pool.
 *
 *   q, o         [total_q, Hq, d] bf16, sequences packed: sequence s owns rows
 *                [cu_seqlens[s], cu_seqlens[s+1])
 *   lse          [total_q, Hq] fp32 (may be NULL)
 *   cu_seqlens   [num_seqs + 1] int32, nondecreasing, cu_seqlens[num_seqs] <=
 *                total_q; every q_len = cu_seqlens[s+1] - cu_seqlens[s] <=
 *                max_q_len (max_q_len sizes the grid)
 *   seq_lens     [num_seqs] int32: keys of sequence s (0 <= len <=
 *                max_pages * page_size)
 *   k_cache, v_cache, block_table: as attn_paged_decode.
 *
 * Query i of sequence s sits at position seq_lens[s] - q_len + i: with causal
 * = 1 it sees keys j <= that position (the bottom-right alignment of
 * attn_fwd), with causal = 0 all keys.  A row with no visible key gets O = 0,
 * lse = -inf.  Supported: d in {64, 128}, page_size in {8, 16, 32, 64},
 * Hq % Hkv == 0, num_pages_total * Hkv < 2^31 (else TA_ERR_UNSUPPORTED: the
 * copies address a (page, KV head) block by one 32-bit coordinate).  Keys
 * are read a page at a time: the rows of a sequence's last page past its
 * length, and physical page 0 (read in place of pages past the sequence),
 * are loaded and given zero weight.  They may hold any finite values, but
 * not NaN or infinity (0 * inf is NaN): zero a pool allocated uninitialised
 * once.
 * Out-of-range lengths, offsets and table entries are clamped
 * on the device (never dereferenced) and flagged in the library status word
 * (ta_device_status).  Allocates nothing.
 */
ta_status attn_paged_prefill(const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_table, const int32_t *cu_seqlens, const int32_t *seq_lens,
                             int page_size, int num_seqs, int total_q, int max_q_len, int Hq, int Hkv, int d,
                             int max_pages, int num_pages_total, float scale, int causal, void *o,
                             float *lse, ta_stream_t stream);

/*
 * attn_lse_merge - merge one partial attention result into an accumulator.
 * A partial is the attention of a set of rows over one block of keys: its
 * output normalised over that block and the block's lse.  Blocks combine
 * exactly by their lse (FlashAttention optimisation article, section 3.2.2:
 * the result does not depend on how keys are blocked), which is how the ring
 * schedule of the LLM-inference article (section 4.1) assembles each device's
 * output from one block per hop.
 *
 *   acc_o     [rows, d] fp32, 16-byte aligned (read unless first, written)
 *   acc_lse   [rows] fp32 (read unless first, written)
 *   part_o    [rows, d] bf16, 8-byte aligned (e.g. attn_fwd's o)
 *   part_lse  [rows] fp32 (attn_fwd's lse; -inf = no visible key)
 *   first     1: acc = part; 0: acc = merge(acc, part):
 *             lse = log(e^lse_acc + e^lse_part),
 *             o = e^(lse_acc - lse) o_acc + e^(lse_part - lse) o_part
 * Rows where both sides are -inf stay O = 0, lse = -inf.  d in {64, 128}.
 */
ta_status attn_lse_merge(float *acc_o, float *acc_lse, const void *part_o, const float *part_lse,
                         int64_t rows, int d, int first, ta_stream_t stream);

/*
 * attn_lse_merge_finish - the accumulator's output as bf16: out [rows, d]
 * (8-byte aligned) = round(acc_o).
 */
ta_status attn_lse_merge_finish(const float *acc_o, void *out, int64_t rows, int d, ta_stream_t stream);

/*
 * Bytes of device workspace attn_bwd needs (256-byte multiple): two fp32
 * values per query row, rows padded to a multiple of 128 per head.  Pure
 * host arithmetic; returns 0 for invalid sizes.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Nq);

/*
 * attn_bwd - gradients of attn_fwd by recomputation.  (The kernel-fusion
 * post, section 4, states the strategy: keep only each row's max and
 * normaliser from the forward pass, recompute the Q K^T blocks during the
 * backward pass and stream the gradients; it prints no formulas.  This call
 * computes the chain rule through the softmax:
 *     dV = P^T dO,  dS = P o (dO V^T - rowsum(dO o O)),
 *     dQ = scale dS K,  dK = scale dS^T Q,
 * with P = exp(scale Q K^T [+ mask] - lse) rebuilt tile by tile.)
 *
 *   q, o, dout, dq   [B, Hq,  Nq,  d]  bf16 (o and lse as written by attn_fwd
 *   k, v, dk, dv     [B, Hkv, Nkv, d]  bf16  for the same q, k, v, scale and
 *   lse              [B, Hq,  Nq]      fp32  causal; dout is the gradient of
 *                                            the loss with respect to o)
 *   workspace        >= attn_bwd_workspace_size(B, Hq, Nq) bytes, 256-byte
 *                    aligned; overwritten.
 *
 * dq, dk, dv are written (not accumulated) in bf16.  With grouped heads a KV
 * head's dk and dv sum the contributions of all Hq / Hkv query heads that read
 * it.  Rows with no visible key (lse = -inf) contribute nothing.  Same
 * supported shapes and conventions as attn_fwd; outputs must not overlap the
 * inputs.  Nq == 0 writes dk = dv = 0 and Nkv == 0 writes dq = 0.  The
 * result does not depend on scheduling: no atomics are used.
 */
ta_status attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
                   const float *lse, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                   int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale, int causal,
                   ta_stream_t stream);

/*
 * Bytes of device workspace attn_paged_decode needs for these sizes (256-byte
 * aligned); returns 0 for invalid sizes.  Host arithmetic on the sizes and the
 * current device's SM count (the split plan aims at 8 CTAs per SM; 148 is
 * assumed when no device can be queried), so query it with the device
 * current that the decode call will run on.  Hkv, which the pages' call
 * sketch leaves out, fixes the number of CTAs per split and so the plan.
 */
size_t attn_paged_decode_workspace_size(int num_seqs, int Hq, int Hkv, int d,
                                        int max_pages, int page_size);

/*
 * attn_paged_decode - one query token per sequence against a paged KV cache
 * (PagedAttention-style pool: GPU-optimisation tag page, "PagedAttention";
 * block gather fused with the dot products and the weighted sum of V: paged
 * gather article, sections 2.1-2.4).
 *
 *   q, o         [num_seqs, Hq, d] bf16
 *   lse          [num_seqs, Hq]    fp32 (may be NULL)
 *   k_cache,
 *   v_cache      [num_pages_total, Hkv, page_size, d] bf16
 *   block_table  [num_seqs, max_pages] int32: logical page t of sequence s is
 *                physical page block_table[s][t]; entries past the last page
 *                of a sequence are ignored
 *   seq_lens     [num_seqs] int32, 0 <= len <= max_pages * page_size; token t
 *                of sequence s is row t % page_size of page
 *                block_table[s][t / page_size].  A sequence of length 0 gets
 *                O = 0, lse = -inf.
 *   workspace    >= attn_paged_decode_workspace_size(...) bytes, 256-byte
 *                aligned; holds split partials and the status word.  Must not
 *                be shared by calls that may run concurrently.
 *
 * Supported: d in {64, 128}, page_size in {8, 16, 32, 64}, Hq % Hkv == 0,
 * Hq / Hkv in {1, 2, 4, 8}.  Table entries outside [0, num_pages_total) and
 * lengths outside [0, max_pages * page_size] are clamped on the device (never
 * dereferenced) and flagged in the status word; see attn_paged_decode_check.
 */
ta_status attn_paged_decode(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_table, const int32_t *seq_lens, int page_size,
                            int num_seqs, int Hq, int Hkv, int d, int max_pages,
                            int num_pages_total, float scale, void *o, float *lse,
                            void *workspace, size_t workspace_bytes, ta_stream_t stream);

/*
 * attn_paged_decode_noalloc - attn_paged_decode for callers that cannot
 * allocate device memory.  (The source pages have no counterpart; this is a
 * library convenience.)  Some callers have no way to obtain a workspace: a
 * plugin inside a host framework that owns all device memory and passes the
 * plugin only its inputs and outputs, or code on a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not acceptable.
 *
 * Same arguments, layouts, limits and results as attn_paged_decode, without
 * `workspace`/`workspace_bytes`: the split partials go to a fixed 64 MiB scratch
 * array in the library's own device memory (a file-scope __device__ array;
 * every GPU that loads the library's code holds it until the process exits).
 * The call allocates nothing.  Sizes whose attn_paged_decode_workspace_size
 * exceeds 64 MiB return TA_ERR_UNSUPPORTED before anything is enqueued (the
 * reason is in ta_last_error).  The first call in each CUDA context (on each
 * device, with that device current) looks up the scratch array's device
 * address and caches it under the context's unique id; make that first call
 * before any stream capture.  A context created later (for example after
 * cudaDeviceReset, or a non-primary context the caller makes current) gets
 * its own lookup on its first call, so no stale address is used.  Every call
 * on a device shares the one array: calls that may overlap on the GPU
 * (different streams, no ordering between them) race and give wrong results;
 * serialise them.  The
 * status word that attn_paged_decode_check reads lives in that shared array
 * and is not exposed for this entry point; bad table entries and lengths are
 * still clamped on the device.
 */
ta_status attn_paged_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *block_table, const int32_t *seq_lens, int page_size,
                                    int num_seqs, int Hq, int Hkv, int d, int max_pages,
                                    int num_pages_total, float scale, void *o, float *lse,
                                    ta_stream_t stream);

/*
 * Checked mode for paged decode: waits for `stream`, reads the status word the
 * last attn_paged_decode wrote into `workspace`, stores it in *flags (host
 * pointer, may be NULL) and returns TA_ERR_BAD_BLOCK_TABLE or
 * TA_ERR_DEVICE_TIMEOUT if a bit is set, else TA_OK.  Synchronises the stream.
 */
ta_status attn_paged_decode_check(const void *workspace, unsigned *flags, ta_stream_t stream);

/*
 * Test/diagnostic export: writes the logical K and V rows of (seq, hkv) to
 * k_out/v_out [max_pages * page_size, d] bf16 (rows >= seq_lens[seq] are left
 * untouched).  The rows are gathered split by split and chunk by chunk with
 * the device functions both attn_paged_decode split kernels use: the split's
 * block-table entries staged in shared memory, then one bulk copy per
 * (page, KV head) of each 64-token chunk.  Same layouts and limits as
 * attn_paged_decode; an entry outside the pool reads physical page 0 and is
 * flagged in the library status word (ta_device_status), as in decode.
 */
ta_status attn_paged_gather_debug(const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, const int32_t *seq_lens,
                                  int seq, int hkv, int page_size, int Hkv, int d, int max_pages,
                                  int num_pages_total, void *k_out, void *v_out, ta_stream_t stream);

/*
 * Library-wide device status word of the current device (bounded-wait
 * timeouts of attn_fwd, gather-debug flags).  Synchronises the device, stores
 * the word in *flags (host pointer, may be NULL), clears it if `reset` is
 * non-zero, and returns TA_ERR_DEVICE_TIMEOUT / TA_ERR_BAD_BLOCK_TABLE if the
 * corresponding bit was set, else TA_OK.
 */
ta_status ta_device_status(unsigned *flags, int reset);

/*
 * Self-test of the bounded waits: launches one CTA that waits on an mbarrier
 * nothing will ever complete, with a limit of `limit_us` microseconds
 * (1..1000000).  The wait gives up, sets TA_DEV_TIMEOUT in the library status
 * word and the kernel exits normally; the context stays usable.
 */
ta_status ta_selftest_bounded_wait(unsigned limit_us, ta_stream_t stream);

/*
 * Test/diagnostic export: y[i] = 2^x[i] for i < n as computed by the FMA-pipe
 * exponential that the FP8 prefill uses for part of its softmax weights
 * (exp((s - m) * scale) with the max subtracted, FlashAttention optimisation
 * article, online softmax section), in place of the MUFU unit.  x and y are
 * device fp32 arrays of n elements (4-byte aligned; they may be the same
 * array); n >= 0, odd n allowed.  Within x >= -125 the maximum relative error is 7.5e-5;
 * below -125, and for NaN inputs, the result is 2^-125.  Returns
 * TA_ERR_INVALID_ARG for n < 0 or a null or misaligned pointer with n > 0,
 * TA_ERR_CUDA if the launch fails.  Asynchronous on `stream`; allocates
 * nothing.
 */
ta_status ta_exp2_poly_debug(const float *x, float *y, int64_t n, ta_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TILEDATTN_H */
