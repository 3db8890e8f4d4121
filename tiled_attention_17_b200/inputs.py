"""Seeded synthetic inputs for the attention workloads.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle's
tests.  It holds no attention arithmetic: it only draws N(0, 1) numbers, rounds
them to bfloat16 bit patterns (or quantises them to FP8 E4M3 codes with a
per-tensor scale), and lays out the paged KV pool and its block table.  Everything is a deterministic function of the seed.

Workloads (shapes and value recipes of the fused-attention pages: FlashAttention
optimisation article, sections 2.1 and 3.1 for N=4096/d=128; the Gemini 3 Flash
kernel-fusion post, "traditional attention" for N=16384 with 8 heads; the paged
gather article, section 2 for block-table gathers):

  tiny     B=1, H=1, N=256, d=64, non-causal
  causal   B=4, Hq=Hkv=16, N=4096, d=128, causal
  long     B=1, Hq=Hkv=8, N=16384, d=128, non-causal, every 64th key row x4
  gqa      B=2, Hq=32, Hkv=8, N=8192, d=128, causal (4 query heads per KV head)
  decode   64 sequences x 1 query, Hq=32, Hkv=8, d=128, 16-token pages,
           lengths uniform on {512..32768}, pages at a seeded permutation of
           the pool's physical slots

Values are float32 N(0,1) from numpy's PCG64, rounded to bfloat16 with
round-to-nearest-even; arrays of bfloat16 are carried as uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

SEED_BASE = 1700


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed_words, n: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(list(seed_words)))
    return f32_to_bf16_bits(rng.standard_normal(n, dtype=np.float32))


def _normal_bf16_chunked(seed_words, n: int, chunk: int = 1 << 22, threads: int | None = None) -> np.ndarray:
    """N(0,1) bf16 bits, generated in independently seeded chunks (parallel)."""
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + chunk - 1) // chunk

    def work(c):
        lo = c * chunk
        hi = min(n, lo + chunk)
        out[lo:hi] = _normal_bf16(list(seed_words) + [c], hi - lo)

    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(nchunks)))
    return out


# --------------------------------------------------------------------------
# Prefill (contiguous) workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    d: int
    causal: bool
    peak_rows_every: int = 0   # if >0: key rows j % peak_rows_every == 0 are scaled
    peak_factor: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


PREFILL_CONFIGS = {
    "tiny": PrefillConfig("tiny", 1, 1, 1, 256, 256, 64, False),
    "causal": PrefillConfig("causal", 4, 16, 16, 4096, 4096, 128, True),
    "long": PrefillConfig("long", 1, 8, 8, 16384, 16384, 128, False, 64, 4.0),
    "gqa": PrefillConfig("gqa", 2, 32, 8, 8192, 8192, 128, True),
}
CONFIG_SEEDS = {"tiny": SEED_BASE + 1, "causal": SEED_BASE + 2, "long": SEED_BASE + 3,
                "gqa": SEED_BASE + 4, "decode": SEED_BASE + 5}


def prefill_inputs(cfg: PrefillConfig, seed: int | None = None):
    """Return (q, k, v) as uint16 bf16 bit arrays shaped [B,H,N,d]."""
    seed = CONFIG_SEEDS.get(cfg.name, SEED_BASE) if seed is None else seed
    nq = cfg.B * cfg.Hq * cfg.Nq * cfg.d
    nk = cfg.B * cfg.Hkv * cfg.Nkv * cfg.d
    q = _normal_bf16_chunked([seed, 0], nq).reshape(cfg.B, cfg.Hq, cfg.Nq, cfg.d)
    if cfg.peak_rows_every:
        rng_k = _chunked_f32([seed, 1], nk).reshape(cfg.B, cfg.Hkv, cfg.Nkv, cfg.d)
        rng_k[:, :, ::cfg.peak_rows_every, :] *= np.float32(cfg.peak_factor)
        k = f32_to_bf16_bits(rng_k.reshape(-1)).reshape(rng_k.shape)
        del rng_k
    else:
        k = _normal_bf16_chunked([seed, 1], nk).reshape(cfg.B, cfg.Hkv, cfg.Nkv, cfg.d)
    v = _normal_bf16_chunked([seed, 2], nk).reshape(cfg.B, cfg.Hkv, cfg.Nkv, cfg.d)
    return q, k, v


def _chunked_f32(seed_words, n: int, chunk: int = 1 << 22) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + chunk - 1) // chunk

    def work(c):
        lo = c * chunk
        hi = min(n, lo + chunk)
        rng = np.random.Generator(np.random.PCG64(list(seed_words) + [c]))
        out[lo:hi] = rng.standard_normal(hi - lo, dtype=np.float32)

    with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(nchunks)))
    return out


def grad_output(shape, seed: int) -> np.ndarray:
    """Seeded loss gradient dO ~ N(0, 1) as bf16 bits (backward-pass inputs)."""
    n = int(np.prod(shape))
    return f32_to_bf16_bits(_chunked_f32([seed, 0xD0], n).reshape(shape))


def random_prefill(B, Hq, Hkv, Nq, Nkv, d, seed, scale_k_rows_every=0, factor=1.0):
    """Small ad-hoc prefill inputs (tests): (q, k, v) uint16 bf16 bits."""
    cfg = PrefillConfig("adhoc", B, Hq, Hkv, Nq, Nkv, d, False, scale_k_rows_every, factor)
    return prefill_inputs(cfg, seed)


# --------------------------------------------------------------------------
# FP8 (E4M3) prefill inputs
# --------------------------------------------------------------------------

E4M3_MAX = 448.0   # largest finite OCP E4M3 ("e4m3fn") magnitude


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values (|x| <= 448) to OCP E4M3 codes (nearest, ties to
    even) with torch's float8_e4m3fn conversion; return uint8 codes."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quantize_e4m3(x: np.ndarray):
    """Per-tensor quantisation: descale = amax / 448 (float32) and codes =
    e4m3(x / descale), so descale * e4m3(code) approximates x."""
    amax = float(np.max(np.abs(x))) if x.size else 1.0
    descale = np.float32(amax / E4M3_MAX if amax > 0 else 1.0)
    codes = f32_to_e4m3_bits(np.clip(x / descale, -E4M3_MAX, E4M3_MAX).astype(np.float32))
    return codes, float(descale)


def random_prefill_fp8(B, Hq, Hkv, Nq, Nkv, d, seed):
    """FP8 prefill inputs: the float32 N(0, 1) draws of prefill_inputs (same
    seed streams), each tensor quantised to E4M3 with its own descale.
    Returns (q8, k8, v8, (q_descale, k_descale, v_descale)), codes as uint8."""
    out, ds = [], []
    for word, shape in ((0, (B, Hq, Nq, d)), (1, (B, Hkv, Nkv, d)), (2, (B, Hkv, Nkv, d))):
        x = _chunked_f32([seed, word], int(np.prod(shape)))
        codes, descale = quantize_e4m3(x)
        out.append(codes.reshape(shape))
        ds.append(descale)
    return out[0], out[1], out[2], tuple(ds)


def fp8_integer_score_inputs(B, Hq, Hkv, Nq, Nkv, d, seed, nnz=3):
    """FP8 inputs whose scores q.k are small integers: every Q and K row has
    `nnz` entries of +-1 at seeded positions (zeros elsewhere), so |q.k| <= nnz;
    V is N(0, 1) quantised per tensor.  With scale = ln 2 every softmax weight
    relative to any score of the row is an exact power of two, which FP8
    represents exactly.  Returns (q8, k8, v8, v_descale)."""
    rng = np.random.Generator(np.random.PCG64([seed, 0xF8]))

    def sparse_rows(rows):
        x = np.zeros((rows, d), dtype=np.float32)
        for r in range(rows):
            cols = rng.choice(d, size=nnz, replace=False)
            x[r, cols] = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=nnz)
        return f32_to_e4m3_bits(x)

    q8 = sparse_rows(B * Hq * Nq).reshape(B, Hq, Nq, d)
    k8 = sparse_rows(B * Hkv * Nkv).reshape(B, Hkv, Nkv, d)
    v8, dv = quantize_e4m3(_chunked_f32([seed, 2], B * Hkv * Nkv * d))
    return q8, k8, v8.reshape(B, Hkv, Nkv, d), dv


# --------------------------------------------------------------------------
# Paged decode workload
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str = "decode"
    num_seqs: int = 64
    Hq: int = 32
    Hkv: int = 8
    d: int = 128
    page_size: int = 16
    len_lo: int = 512
    len_hi: int = 32768

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def max_pages(self) -> int:
        return (self.len_hi + self.page_size - 1) // self.page_size


DECODE_CONFIG = DecodeConfig()


@dataclasses.dataclass
class PagedInputs:
    cfg: DecodeConfig
    seed: int
    q: np.ndarray            # [S, Hq, d] bf16 bits
    seq_lens: np.ndarray     # [S] int32
    block_table: np.ndarray  # [S, max_pages] int32, -1 beyond each sequence
    num_pages_total: int
    k_cache: np.ndarray | None = None   # [P_tot, Hkv, page, d] bf16 bits
    v_cache: np.ndarray | None = None


PAGE_CHUNK = 64   # pages per independently seeded chunk of the pool


def pool_pages(cfg: DecodeConfig, seed: int, which: int, first: int, count: int) -> np.ndarray:
    """Pages [first, first+count) of the K (which=1) or V (which=2) pool.

    The pool is generated in independently seeded chunks of PAGE_CHUNK pages,
    so any page can be regenerated on its own.
    """
    per_page = cfg.Hkv * cfg.page_size * cfg.d
    out = np.empty((count, per_page), dtype=np.uint16)
    p = first
    while p < first + count:
        c = p // PAGE_CHUNK
        c_lo = c * PAGE_CHUNK
        chunk = _normal_bf16([seed, 10 + which, c], PAGE_CHUNK * per_page).reshape(PAGE_CHUNK, per_page)
        hi = min(first + count, c_lo + PAGE_CHUNK)
        out[p - first:hi - first] = chunk[p - c_lo:hi - c_lo]
        p = hi
    return out.reshape(count, cfg.Hkv, cfg.page_size, cfg.d)


def _pool(cfg: DecodeConfig, seed: int, which: int, total: int) -> np.ndarray:
    per_page = cfg.Hkv * cfg.page_size * cfg.d
    out = np.empty((total, per_page), dtype=np.uint16)
    nchunks = (total + PAGE_CHUNK - 1) // PAGE_CHUNK

    def work(c):
        lo = c * PAGE_CHUNK
        hi = min(total, lo + PAGE_CHUNK)
        chunk = _normal_bf16([seed, 10 + which, c], PAGE_CHUNK * per_page).reshape(PAGE_CHUNK, per_page)
        out[lo:hi] = chunk[:hi - lo]

    with ThreadPoolExecutor(min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(work, range(nchunks)))
    return out.reshape(total, cfg.Hkv, cfg.page_size, cfg.d)


def paged_inputs(cfg: DecodeConfig = DECODE_CONFIG, seed: int | None = None, with_pool: bool = True,
                 seq_lens: np.ndarray | None = None, extra_pages: int = 0) -> PagedInputs:
    """Build the paged decode workload.

    Lengths are uniform integers on [len_lo, len_hi] (inclusive) unless given.
    The pool holds exactly the pages the sequences use (plus `extra_pages`
    unused slots); the logical page t of sequence s sits at physical slot
    perm[offset_s + t] for one seeded permutation of all slots.  Table entries
    past a sequence's last page are -1.
    """
    seed = CONFIG_SEEDS["decode"] if seed is None else seed
    rng = np.random.Generator(np.random.PCG64([seed, 0]))
    if seq_lens is None:
        seq_lens = rng.integers(cfg.len_lo, cfg.len_hi, size=cfg.num_seqs, endpoint=True)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    assert seq_lens.shape == (cfg.num_seqs,)
    npages = (seq_lens.astype(np.int64) + cfg.page_size - 1) // cfg.page_size
    total = int(npages.sum()) + extra_pages
    perm = np.random.Generator(np.random.PCG64([seed, 1])).permutation(total).astype(np.int32)
    table = np.full((cfg.num_seqs, cfg.max_pages), -1, dtype=np.int32)
    off = 0
    for s in range(cfg.num_seqs):
        n = int(npages[s])
        table[s, :n] = perm[off:off + n]
        off += n
    q = _normal_bf16([seed, 2], cfg.num_seqs * cfg.Hq * cfg.d).reshape(cfg.num_seqs, cfg.Hq, cfg.d)
    inp = PagedInputs(cfg, seed, q, seq_lens, table, max(total, 1))
    if with_pool:
        inp.k_cache = _pool(cfg, seed, 1, inp.num_pages_total)
        inp.v_cache = _pool(cfg, seed, 2, inp.num_pages_total)
    return inp


# --------------------------------------------------------------------------
# Varlen prefill over the paged cache
# --------------------------------------------------------------------------

@dataclasses.dataclass
class PagedPrefillInputs:
    q: np.ndarray            # [total_q, Hq, d] bf16 bits, packed by cu_seqlens
    cu_seqlens: np.ndarray   # [S + 1] int32
    seq_lens: np.ndarray     # [S] int32 keys per sequence (prefix + new tokens)
    block_table: np.ndarray  # [S, max_pages] int32, -1 beyond each sequence
    k_cache: np.ndarray      # [P, Hkv, page, d] bf16 bits
    v_cache: np.ndarray
    max_q_len: int


def paged_prefill_inputs(q_lens, kv_lens, Hq: int, Hkv: int, d: int, page_size: int, seed: int,
                         extra_pages: int = 2) -> PagedPrefillInputs:
    """Seeded varlen batch: sequence s has q_lens[s] new queries and kv_lens[s]
    keys in total; its pages sit at a seeded permutation of the pool's slots."""
    q_lens = np.asarray(q_lens, dtype=np.int32)
    kv_lens = np.asarray(kv_lens, dtype=np.int32)
    S = q_lens.size
    cu = np.zeros(S + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    npages = (kv_lens.astype(np.int64) + page_size - 1) // page_size
    total = int(npages.sum()) + extra_pages
    max_pages = max(int(npages.max()) if S else 1, 1)
    perm = np.random.Generator(np.random.PCG64([seed, 1])).permutation(total).astype(np.int32)
    table = np.full((S, max_pages), -1, dtype=np.int32)
    off = 0
    for s in range(S):
        n = int(npages[s])
        table[s, :n] = perm[off:off + n]
        off += n
    T = int(cu[-1])
    q = _normal_bf16([seed, 2], max(T, 1) * Hq * d)[:T * Hq * d].reshape(T, Hq, d)
    per = total * Hkv * page_size * d
    k = _normal_bf16_chunked([seed, 3], per).reshape(total, Hkv, page_size, d)
    v = _normal_bf16_chunked([seed, 4], per).reshape(total, Hkv, page_size, d)
    return PagedPrefillInputs(q, cu, kv_lens, table, k, v, int(q_lens.max()) if S else 0)
