"""ctypes binding of libtiledattn.so (argument marshalling only).

Every function here passes device pointers, sizes and the CUDA stream through
to the C ABI declared in include/tiledattn.h; all computation happens in the
library's kernels.  There is no fallback: if the shared object cannot be
loaded, every call raises.

Functions with the C names take raw integers (device pointers) or torch
tensors (their data_ptr() is passed).  `attention()` and `paged_decode()` are
conveniences that allocate outputs with torch and call the C entry points.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtiledattn.so")

TA_OK = 0
STATUS_NAMES = {0: "TA_OK", 1: "TA_ERR_INVALID_ARG", 2: "TA_ERR_UNSUPPORTED", 3: "TA_ERR_CUDA",
                4: "TA_ERR_BAD_BLOCK_TABLE", 5: "TA_ERR_DEVICE_TIMEOUT"}
TA_DEV_TIMEOUT = 1
TA_DEV_BAD_BLOCK_TABLE = 2
TA_DEV_BAD_SEQ_LEN = 4

EXPORTS = ["ta_status_string", "ta_version", "ta_last_error", "attn_fwd", "attn_fwd_fp8", "attn_bwd_workspace_size",
           "attn_bwd",
           "attn_paged_prefill", "attn_lse_merge", "attn_lse_merge_finish",
           "attn_paged_decode_workspace_size",
           "attn_paged_decode", "attn_paged_decode_noalloc", "attn_paged_decode_check", "attn_paged_gather_debug",
           "ta_device_status", "ta_selftest_bounded_wait", "ta_exp2_poly_debug"]


class TiledAttnError(RuntimeError):
    def __init__(self, fn, code, detail=""):
        self.code = code
        msg = f"{fn} returned {STATUS_NAMES.get(code, code)}"
        super().__init__(msg + (f": {detail}" if detail else ""))


_lib = None


def load(path: str | None = None):
    """Load (once) and return the ctypes handle of libtiledattn.so."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libtiledattn.so not found at {p}; build it with "
                           f"`python -m tiled_attention_17_b200.build`")
    L = ctypes.CDLL(p)
    vp, i32, f32, sz, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint
    L.ta_status_string.argtypes = [i32]
    L.ta_status_string.restype = ctypes.c_char_p
    L.ta_version.restype = i32
    L.ta_last_error.restype = ctypes.c_char_p
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp] + [i32] * 6 + [f32, i32, vp]
    L.attn_fwd.restype = i32
    L.attn_fwd_fp8.argtypes = [vp, vp, vp, f32, f32, f32, vp, vp] + [i32] * 6 + [f32, i32, vp]
    L.attn_fwd_fp8.restype = i32
    L.attn_paged_prefill.argtypes = [vp] * 6 + [i32] * 9 + [f32, i32, vp, vp, vp]
    L.attn_paged_prefill.restype = i32
    i64 = ctypes.c_int64
    L.attn_lse_merge.argtypes = [vp, vp, vp, vp, i64, i32, i32, vp]
    L.attn_lse_merge.restype = i32
    L.attn_lse_merge_finish.argtypes = [vp, vp, i64, i32, vp]
    L.attn_lse_merge_finish.restype = i32
    L.attn_bwd_workspace_size.argtypes = [i32] * 3
    L.attn_bwd_workspace_size.restype = sz
    L.attn_bwd.argtypes = [vp] * 10 + [sz] + [i32] * 6 + [f32, i32, vp]
    L.attn_bwd.restype = i32
    L.attn_paged_decode_workspace_size.argtypes = [i32] * 6
    L.attn_paged_decode_workspace_size.restype = sz
    L.attn_paged_decode.argtypes = [vp, vp, vp, vp, vp] + [i32] * 7 + [f32, vp, vp, vp, sz, vp]
    L.attn_paged_decode.restype = i32
    L.attn_paged_decode_noalloc.argtypes = [vp, vp, vp, vp, vp] + [i32] * 7 + [f32, vp, vp, vp]
    L.attn_paged_decode_noalloc.restype = i32
    L.attn_paged_decode_check.argtypes = [vp, ctypes.POINTER(u32), vp]
    L.attn_paged_decode_check.restype = i32
    L.attn_paged_gather_debug.argtypes = [vp, vp, vp, vp] + [i32] * 7 + [vp, vp, vp]
    L.attn_paged_gather_debug.restype = i32
    L.ta_device_status.argtypes = [ctypes.POINTER(u32), i32]
    L.ta_device_status.restype = i32
    L.ta_selftest_bounded_wait.argtypes = [u32, vp]
    L.ta_selftest_bounded_wait.restype = i32
    L.ta_exp2_poly_debug.argtypes = [vp, vp, i64, vp]
    L.ta_exp2_poly_debug.restype = i32
    if path is None:
        _lib = L
    return L


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, code):
    if code != TA_OK:
        raise TiledAttnError(fn, code, ta_last_error())


# ---------------------------------------------------------------------------
# C-named entry points
# ---------------------------------------------------------------------------

def ta_status_string(code: int) -> str:
    return load().ta_status_string(code).decode()


def ta_version() -> int:
    return load().ta_version()


def ta_last_error() -> str:
    return load().ta_last_error().decode()


def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, stream=None, check=True) -> int:
    code = load().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nkv, d,
                           float(scale), int(causal), _stream(stream))
    if check:
        _check("attn_fwd", code)
    return code


def attn_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal,
                 stream=None, check=True) -> int:
    code = load().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), float(q_descale), float(k_descale), float(v_descale),
                               _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nkv, d, float(scale), int(causal), _stream(stream))
    if check:
        _check("attn_fwd_fp8", code)
    return code


def attn_paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, page_size, num_seqs, total_q,
                       max_q_len, Hq, Hkv, d, max_pages, num_pages_total, scale, causal, o, lse, stream=None,
                       check=True) -> int:
    code = load().attn_paged_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cu_seqlens),
                                     _ptr(seq_lens), page_size, num_seqs, total_q, max_q_len, Hq, Hkv, d, max_pages,
                                     num_pages_total, float(scale), int(causal), _ptr(o), _ptr(lse),
                                     _stream(stream))
    if check:
        _check("attn_paged_prefill", code)
    return code


def attn_lse_merge(acc_o, acc_lse, part_o, part_lse, rows, d, first, stream=None, check=True) -> int:
    code = load().attn_lse_merge(_ptr(acc_o), _ptr(acc_lse), _ptr(part_o), _ptr(part_lse), int(rows), d, int(first),
                                 _stream(stream))
    if check:
        _check("attn_lse_merge", code)
    return code


def attn_lse_merge_finish(acc_o, out, rows, d, stream=None, check=True) -> int:
    code = load().attn_lse_merge_finish(_ptr(acc_o), _ptr(out), int(rows), d, _stream(stream))
    if check:
        _check("attn_lse_merge_finish", code)
    return code


def attn_bwd_workspace_size(B, Hq, Nq) -> int:
    return load().attn_bwd_workspace_size(B, Hq, Nq)


def attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, Nq, Nkv, d, scale,
             causal, stream=None, check=True) -> int:
    code = load().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                           _ptr(workspace), int(workspace_bytes), B, Hq, Hkv, Nq, Nkv, d, float(scale), int(causal),
                           _stream(stream))
    if check:
        _check("attn_bwd", code)
    return code


def attn_paged_decode_workspace_size(num_seqs, Hq, Hkv, d, max_pages, page_size) -> int:
    return load().attn_paged_decode_workspace_size(num_seqs, Hq, Hkv, d, max_pages, page_size)


def attn_paged_decode(q, k_cache, v_cache, block_table, seq_lens, page_size, num_seqs, Hq, Hkv, d,
                      max_pages, num_pages_total, scale, o, lse, workspace, workspace_bytes,
                      stream=None, check=True) -> int:
    code = load().attn_paged_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                    page_size, num_seqs, Hq, Hkv, d, max_pages, num_pages_total, float(scale),
                                    _ptr(o), _ptr(lse), _ptr(workspace), int(workspace_bytes), _stream(stream))
    if check:
        _check("attn_paged_decode", code)
    return code


def attn_paged_decode_noalloc(q, k_cache, v_cache, block_table, seq_lens, page_size, num_seqs, Hq, Hkv, d,
                              max_pages, num_pages_total, scale, o, lse, stream=None, check=True) -> int:
    """attn_paged_decode without a workspace argument, for callers that cannot
    allocate device memory: the library uses its own fixed 64 MiB scratch array
    (shared by all calls on a device; overlapping calls race)."""
    code = load().attn_paged_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                            _ptr(seq_lens), page_size, num_seqs, Hq, Hkv, d, max_pages,
                                            num_pages_total, float(scale), _ptr(o), _ptr(lse), _stream(stream))
    if check:
        _check("attn_paged_decode_noalloc", code)
    return code


def attn_paged_decode_check(workspace, stream=None):
    flags = ctypes.c_uint(0)
    code = load().attn_paged_decode_check(_ptr(workspace), ctypes.byref(flags), _stream(stream))
    return code, flags.value


def attn_paged_gather_debug(k_cache, v_cache, block_table, seq_lens, seq, hkv, page_size, Hkv, d, max_pages,
                            num_pages_total, k_out, v_out, stream=None, check=True) -> int:
    code = load().attn_paged_gather_debug(_ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                          seq, hkv, page_size, Hkv, d, max_pages, num_pages_total,
                                          _ptr(k_out), _ptr(v_out), _stream(stream))
    if check:
        _check("attn_paged_gather_debug", code)
    return code


def ta_device_status(reset: bool = True):
    flags = ctypes.c_uint(0)
    code = load().ta_device_status(ctypes.byref(flags), int(reset))
    return code, flags.value


def ta_selftest_bounded_wait(limit_us: int, stream=None) -> int:
    return load().ta_selftest_bounded_wait(int(limit_us), _stream(stream))


def ta_exp2_poly_debug(x, y, n: int, stream=None, check: bool = True) -> int:
    code = load().ta_exp2_poly_debug(_ptr(x), _ptr(y), int(n), _stream(stream))
    if check:
        _check("ta_exp2_poly_debug", code)
    return code


# ---------------------------------------------------------------------------
# torch conveniences (allocate outputs, then call the C entry points)
# ---------------------------------------------------------------------------

def attention(q, k, v, causal: bool, scale: float | None = None, out=None, lse=None, stream=None):
    """q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] bf16 CUDA tensors -> (o, lse)."""
    import torch
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
    if scale is None:
        scale = d ** -0.5
    o = out if out is not None else torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, stream)
    return o, lse


def attention_fp8(q, k, v, descale, causal: bool, scale: float | None = None, out=None, lse=None, stream=None):
    """q [B,Hq,Nq,128], k/v [B,Hkv,Nkv,128] contiguous CUDA tensors of E4M3
    codes (torch.float8_e4m3fn or uint8); descale = (q_descale, k_descale,
    v_descale) -> (o bf16, lse fp32)."""
    import torch
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    for t in (q, k, v):
        if t.dtype not in (torch.float8_e4m3fn, torch.uint8) or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous float8_e4m3fn (or uint8) CUDA tensors")
    if scale is None:
        scale = d ** -0.5
    o = out if out is not None else torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    dq, dk, dv = descale
    attn_fwd_fp8(q, k, v, dq, dk, dv, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool, scale: float | None = None, workspace=None,
                       stream=None):
    """Gradients (dq, dk, dv) of `attention` for the loss gradient dout (all bf16
    CUDA tensors; o and lse from the forward call with the same arguments)."""
    import torch
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = k.shape
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, o, dout must be contiguous bf16 CUDA tensors")
    if scale is None:
        scale = d ** -0.5
    ws_bytes = attn_bwd_workspace_size(B, Hq, Nq)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, workspace, workspace.numel(), B, Hq, Hkv, Nq, Nkv, d, scale,
             causal, stream)
    return dq, dk, dv


def paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, max_q_len: int, causal: bool,
                  scale: float | None = None, out=None, lse=None, stream=None):
    """q [total_q, Hq, d] packed by cu_seqlens [S+1] (int32, device); caches
    [P, Hkv, page, d]; block_table [S, max_pages]; seq_lens [S] -> (o, lse)."""
    import torch
    T, Hq, d = q.shape
    P, Hkv, ps, _ = k_cache.shape
    S = seq_lens.shape[0]
    if scale is None:
        scale = d ** -0.5
    o = out if out is not None else torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    attn_paged_prefill(q, k_cache, v_cache, block_table, cu_seqlens, seq_lens, ps, S, T, max_q_len, Hq, Hkv, d,
                       block_table.shape[1], P, scale, causal, o, lse, stream)
    return o, lse


def paged_decode(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None, workspace=None,
                 out=None, lse=None, stream=None):
    """q [S,Hq,d]; caches [P,Hkv,page,d] bf16; block_table [S,max_pages] int32; seq_lens [S] int32."""
    import torch
    S, Hq, d = q.shape
    P, Hkv, ps, _ = k_cache.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = d ** -0.5
    ws_bytes = attn_paged_decode_workspace_size(S, Hq, Hkv, d, max_pages, ps)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=q.device)
    o = out if out is not None else torch.empty_like(q)
    if lse is None:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    attn_paged_decode(q, k_cache, v_cache, block_table, seq_lens, ps, S, Hq, Hkv, d, max_pages, P, scale,
                      o, lse, workspace, workspace.numel(), stream)
    return o, lse, workspace
