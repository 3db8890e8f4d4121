"""The C-ABI library on the host (no GPU needed): it builds, loads, exports
every entry point the header declares, and rejects bad arguments before any
CUDA call."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tiledattn.h")


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_17_b200 import binding, build
    build.build()
    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) - {"defined"})


def test_header_functions_exported(lib):
    import ctypes
    L = lib.load()
    names = declared_functions()
    assert set(lib.EXPORTS) == set(names), (names, lib.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
        assert isinstance(getattr(L, n), ctypes._CFuncPtr)


def declared_signatures():
    """{name: [parameter types]} parsed from the header's prototypes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b([a-z_][a-z0-9_ ]*?[ *]+)([a-z_][a-z0-9_]*)\s*\(([^;{]*?)\)\s*;", text):
        name, params = m.group(2), " ".join(m.group(3).split())
        if name == "defined":
            continue
        out[name] = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
    return out


def test_binding_argtypes_match_header(lib):
    # every ctypes prototype has the header's parameter count, and pointer /
    # integer / float / size_t kinds in the same places
    import ctypes
    L = lib.load()
    sigs = declared_signatures()
    assert set(sigs) == set(lib.EXPORTS)
    for name, params in sigs.items():
        argtypes = getattr(L, name).argtypes or []
        assert len(argtypes) == len(params), (name, len(argtypes), params)
        for p, t in zip(params, argtypes):
            if "*" in p or p.startswith("ta_stream_t"):
                assert t is ctypes.c_void_p or issubclass(t, ctypes._Pointer) or t is ctypes.c_char_p, (name, p, t)
            elif p.startswith("float"):
                assert t is ctypes.c_float, (name, p, t)
            elif p.startswith("size_t"):
                assert t is ctypes.c_size_t, (name, p, t)
            elif p.startswith("int64_t"):
                assert t is ctypes.c_int64, (name, p, t)
            else:
                assert t in (ctypes.c_int, ctypes.c_uint), (name, p, t)


def test_status_strings(lib):
    assert lib.ta_status_string(0) == "TA_OK"
    assert lib.ta_status_string(4) == "TA_ERR_BAD_BLOCK_TABLE"
    assert lib.ta_status_string(99) == "TA_ERR_UNKNOWN"
    assert lib.ta_version() == 10000


def code(lib, c):
    return lib.STATUS_NAMES[c]


def test_attn_fwd_validation(lib):
    a = 256  # any 16-byte-aligned non-null value: rejected before use
    f = lambda *x, **kw: code(lib, lib.attn_fwd(*x, check=False, stream=0, **kw))
    assert f(a, a, a, a, None, 1, 3, 2, 128, 128, 128, 0.1, 0) == "TA_ERR_INVALID_ARG"   # Hq % Hkv
    assert f(a, a, a, a, None, 1, 1, 1, 128, 128, 96, 0.1, 0) == "TA_ERR_UNSUPPORTED"   # head dim
    assert f(a + 2, a, a, a, None, 1, 1, 1, 128, 128, 128, 0.1, 0) == "TA_ERR_INVALID_ARG"  # alignment
    assert f(a, a, a, a, a + 2, 1, 1, 1, 128, 128, 128, 0.1, 0) == "TA_ERR_INVALID_ARG"  # lse alignment
    assert f(a, a, a, a, None, 1, 1, 1, 128, 128, 128, -0.5, 0) == "TA_ERR_UNSUPPORTED"  # negative scale
    assert f(a, a, a, a, None, 1, 1, 1, 128, 128, 128, float("nan"), 0) == "TA_ERR_UNSUPPORTED"
    assert f(a, a, a, a, None, 1, 1, 1, 128, 128, 128, 0.1, 2) == "TA_ERR_INVALID_ARG"   # causal flag
    assert f(a, a, a, a, None, -1, 1, 1, 128, 128, 128, 0.1, 0) == "TA_ERR_INVALID_ARG"  # negative size
    assert f(None, a, a, a, None, 1, 1, 1, 128, 128, 128, 0.1, 0) == "TA_ERR_INVALID_ARG"  # null
    assert f(a, a, a, a, None, 0, 1, 1, 128, 128, 128, 0.1, 0) == "TA_OK"                # empty: no-op
    assert f(None, None, None, None, None, 1, 1, 1, 0, 128, 128, 0.1, 0) == "TA_OK"


def test_attn_fwd_fp8_validation(lib):
    a = 256
    f = lambda *x: code(lib, lib.attn_fwd_fp8(*x, check=False, stream=0))

    def call(q=a, lse=None, dq=0.01, dk=0.02, dv=0.03, B=1, Hq=2, Hkv=1, d=128, scale=0.1, causal=1):
        return f(q, a, a, dq, dk, dv, a, lse, B, Hq, Hkv, 256, 256, d, scale, causal)

    assert call(d=64) == "TA_ERR_UNSUPPORTED"                 # fp8 path: d = 128 only
    assert call(Hq=3, Hkv=2) == "TA_ERR_INVALID_ARG"
    assert call(dq=0.0) == "TA_ERR_INVALID_ARG"               # descales finite and > 0
    assert call(dk=-1.0) == "TA_ERR_INVALID_ARG"
    assert call(dv=float("inf")) == "TA_ERR_INVALID_ARG"
    assert call(dq=1e30, dk=1e30) == "TA_ERR_UNSUPPORTED"     # folded score scale overflows fp32
    assert call(scale=-1.0) == "TA_ERR_UNSUPPORTED"
    assert call(causal=3) == "TA_ERR_INVALID_ARG"
    assert call(q=a + 1) == "TA_ERR_INVALID_ARG"              # 16-byte alignment
    assert call(lse=a + 2) == "TA_ERR_INVALID_ARG"
    assert call(q=None) == "TA_ERR_INVALID_ARG"
    assert call(B=0) == "TA_OK"


def test_decode_validation(lib):
    a = 256
    f = lambda *x: code(lib, lib.attn_paged_decode(*x, check=False, stream=0))
    ws = lib.attn_paged_decode_workspace_size(4, 8, 2, 128, 64, 16)
    good = dict(q=a, kc=a, vc=a, bt=a, sl=a, ps=16, S=4, Hq=8, Hkv=2, d=128, mp=64, P=100)

    def call(**kw):
        g = dict(good, **kw)
        return f(g["q"], g["kc"], g["vc"], g["bt"], g["sl"], g["ps"], g["S"], g["Hq"], g["Hkv"], g["d"],
                 g["mp"], g["P"], 0.1, a, None, a, kw.get("wsb", ws))

    assert call(ps=12) == "TA_ERR_UNSUPPORTED"
    assert call(ps=128) == "TA_ERR_UNSUPPORTED"
    assert call(Hq=6, Hkv=4) == "TA_ERR_INVALID_ARG"
    assert call(Hq=24, Hkv=2) == "TA_ERR_UNSUPPORTED"      # group of 12
    assert call(d=80) == "TA_ERR_UNSUPPORTED"
    assert call(wsb=ws - 1) == "TA_ERR_INVALID_ARG"
    assert call(q=a + 8) == "TA_ERR_INVALID_ARG"
    assert call(bt=a + 2) == "TA_ERR_INVALID_ARG"
    assert call(P=0) == "TA_ERR_INVALID_ARG"
    assert call(S=0) == "TA_OK"


def test_workspace_plan(lib):
    # 64 sequences x 8 KV heads x 2048 pages of 16: 2048-token splits -> 16 splits
    ws = lib.attn_paged_decode_workspace_size(64, 32, 8, 128, 2048, 16)
    rows = 64 * 32 * 16
    assert ws >= rows * 128 * 4 + rows * 4 + 256
    assert ws % 256 == 0
    assert lib.attn_paged_decode_workspace_size(64, 32, 8, 128, 2048, 12) == 0
    assert lib.attn_paged_decode_workspace_size(64, 30, 8, 128, 2048, 16) == 0
    # a single short-batch sequence splits finer to fill the GPU
    ws1 = lib.attn_paged_decode_workspace_size(1, 32, 8, 128, 2048, 16)
    assert ws1 > 1 * 32 * 32 * 128 * 4


def test_gather_debug_validation(lib):
    a = 256
    c = lib.attn_paged_gather_debug(a, a, a, a, 0, 2, 16, 2, 128, 8, 10, a, a, stream=0, check=False)
    assert code(lib, c) == "TA_ERR_INVALID_ARG"     # hkv out of range
    c = lib.attn_paged_gather_debug(a, a, a, a, 0, 0, 16, 2, 96, 8, 10, a, a, stream=0, check=False)
    assert code(lib, c) == "TA_ERR_UNSUPPORTED"


def test_selftest_validation(lib):
    assert code(lib, lib.ta_selftest_bounded_wait(0, stream=0)) == "TA_ERR_INVALID_ARG"
    assert code(lib, lib.ta_selftest_bounded_wait(2_000_000, stream=0)) == "TA_ERR_INVALID_ARG"


def test_exp2_poly_debug_validation(lib):
    # argument checks only: nothing is launched
    assert code(lib, lib.ta_exp2_poly_debug(256, 256, -1, stream=0, check=False)) == "TA_ERR_INVALID_ARG"
    assert code(lib, lib.ta_exp2_poly_debug(None, 256, 8, stream=0, check=False)) == "TA_ERR_INVALID_ARG"
    assert code(lib, lib.ta_exp2_poly_debug(258, 256, 8, stream=0, check=False)) == "TA_ERR_INVALID_ARG"
    assert code(lib, lib.ta_exp2_poly_debug(None, None, 0, stream=0, check=False)) == "TA_OK"


def test_bwd_validation(lib):
    a = 256
    ws = lib.attn_bwd_workspace_size(4, 16, 4096)
    assert ws == 2 * 4 * 16 * 4096 * 4 and ws % 256 == 0
    assert lib.attn_bwd_workspace_size(1, 2, 130) == 2 * 2 * 256 * 4   # rows padded to 128 per head
    assert lib.attn_bwd_workspace_size(1, 0, 128) == 0
    f = lambda *x, **kw: code(lib, lib.attn_bwd(*x, check=False, stream=0, **kw))

    def call(**kw):
        g = dict(q=a, k=a, v=a, o=a, do=a, lse=a, dq=a, dk=a, dv=a, ws=a, wsb=1 << 20,
                 B=1, Hq=2, Hkv=1, Nq=128, Nkv=128, d=128, scale=0.1, causal=1)
        g.update(kw)
        return f(g["q"], g["k"], g["v"], g["o"], g["do"], g["lse"], g["dq"], g["dk"], g["dv"], g["ws"], g["wsb"],
                 g["B"], g["Hq"], g["Hkv"], g["Nq"], g["Nkv"], g["d"], g["scale"], g["causal"])

    assert call(Hq=3, Hkv=2) == "TA_ERR_INVALID_ARG"
    assert call(d=96) == "TA_ERR_UNSUPPORTED"
    assert call(causal=2) == "TA_ERR_INVALID_ARG"
    assert call(scale=-1.0) == "TA_ERR_UNSUPPORTED"
    assert call(dq=a + 8) == "TA_ERR_INVALID_ARG"          # 16-byte alignment
    assert call(lse=None) == "TA_ERR_INVALID_ARG"
    assert call(wsb=16) == "TA_ERR_INVALID_ARG"            # workspace too small
    assert call(ws=a + 16) == "TA_ERR_INVALID_ARG"         # workspace not 256-byte aligned
    assert call(B=0) == "TA_OK"                            # nothing to do, no CUDA call


def test_paged_prefill_validation(lib):
    a = 256
    f = lambda *x, **kw: code(lib, lib.attn_paged_prefill(*x, check=False, stream=0, **kw))

    def call(**kw):
        g = dict(q=a, kc=a, vc=a, bt=a, cu=a, sl=a, ps=16, S=2, T=100, mq=64, Hq=4, Hkv=2, d=128, mp=8, P=20,
                 scale=0.1, causal=1, o=a, lse=None)
        g.update(kw)
        return f(g["q"], g["kc"], g["vc"], g["bt"], g["cu"], g["sl"], g["ps"], g["S"], g["T"], g["mq"], g["Hq"],
                 g["Hkv"], g["d"], g["mp"], g["P"], g["scale"], g["causal"], g["o"], g["lse"])

    assert call(ps=12) == "TA_ERR_UNSUPPORTED"
    assert call(d=80) == "TA_ERR_UNSUPPORTED"
    assert call(Hq=6, Hkv=4) == "TA_ERR_INVALID_ARG"
    assert call(causal=3) == "TA_ERR_INVALID_ARG"
    assert call(q=a + 4) == "TA_ERR_INVALID_ARG"
    assert call(cu=None) == "TA_ERR_INVALID_ARG"
    assert call(lse=a + 2) == "TA_ERR_INVALID_ARG"
    assert call(P=0) == "TA_ERR_INVALID_ARG"
    assert call(P=2 ** 30, Hkv=2, Hq=4) == "TA_ERR_UNSUPPORTED"   # (page, head) blocks past a 32-bit coordinate
    assert call(S=0) == "TA_OK"
    assert call(T=0) == "TA_OK"


def test_merge_validation(lib):
    a = 256
    m = lambda *x: code(lib, lib.attn_lse_merge(*x, stream=0, check=False))
    assert m(a, a, a, a, 16, 80, 0) == "TA_ERR_UNSUPPORTED"
    assert m(a, a, a, a, 16, 128, 2) == "TA_ERR_INVALID_ARG"
    assert m(a + 8, a, a, a, 16, 128, 0) == "TA_ERR_INVALID_ARG"    # fp32 accumulator 16-byte aligned
    assert m(a, a, a + 4, a, 16, 128, 0) == "TA_ERR_INVALID_ARG"    # bf16 partial 8-byte aligned
    assert m(a, a, a, a, -1, 128, 0) == "TA_ERR_INVALID_ARG"
    assert m(a, a, a, a, 0, 128, 0) == "TA_OK"
    fin = lambda *x: code(lib, lib.attn_lse_merge_finish(*x, stream=0, check=False))
    assert fin(a, a, 16, 96) == "TA_ERR_UNSUPPORTED"
    assert fin(a, a + 4, 16, 128) == "TA_ERR_INVALID_ARG"
    assert fin(a, a, 0, 128) == "TA_OK"


def test_header_is_plain_c(tmp_path):
    """include/tiledattn.h compiles as C11 with warnings as errors, and a C
    program linked against libtiledattn.so reaches the host-side paths (no GPU
    needed: argument checks return before any CUDA call)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    from tiled_attention_17_b200 import build as libbuild
    lib = libbuild.build()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "consumer.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "tiledattn.h"
int main(void) {
    void *p = (void *)(size_t)256;   /* aligned, never dereferenced: rejected first */
    if (attn_fwd(p, p, p, p, NULL, 1, 3, 2, 128, 128, 128, 0.1f, 0, NULL) != TA_ERR_INVALID_ARG) return 1;
    if (attn_fwd_fp8(p, p, p, 1.f, 1.f, 1.f, p, NULL, 1, 1, 1, 128, 128, 64, 0.1f, 1, NULL) != TA_ERR_UNSUPPORTED)
        return 2;
    if (attn_bwd_workspace_size(1, 1, 1) == 0) return 3;
    if (strcmp(ta_status_string(TA_OK), "TA_OK") != 0) return 4;
    printf("version %d\n", ta_version());
    return ta_version() > 0 ? 0 : 5;
}
""")
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                    str(src), "-o", str(exe), f"-L{libdir}", "-ltiledattn", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
