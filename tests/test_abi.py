"""The C-ABI library loads and exports every entry point include/moe.h
declares; host-only entry points answer without a GPU."""
import re

import pytest

from expert_streaming_decode_b200 import moe, synth


def test_exports_every_declared_symbol():
    names = moe.declared_symbols()
    assert len(names) >= 14
    missing = [n for n in names if not hasattr(moe.lib, n)]
    assert not missing, missing


def test_host_only_calls():
    assert moe.blob_bytes(2816, 704) == 3345408 == synth.blob_bytes(2816, 704)
    assert moe.blob_bytes(2816, 2112) == 10036224
    assert moe.blob_bytes(512, 64) == synth.blob_bytes(512, 64)
    assert moe.blob_bytes(2816, 700) == 0          # not a multiple of 64
    assert moe.blob_bytes(2816, 1000) == 0         # > 704 and not a multiple of 704
    d = moe.moe_dims(2816, 128, 8, 704, 2112, 64, 16, 1)
    assert moe.lib.moe_cache_state_words(d) == 3 * 128 + 16
    for code in range(-6, 1):
        assert moe.status_str(code) not in ("", "unknown status")
    assert moe.status_str(-99) == "unknown status"


def test_ctx_create_rejects_bad_dims_without_touching_a_gpu():
    import ctypes as C
    h = C.c_void_p()
    bad = moe.moe_dims(2816, 128, 8, 704, 2112, 32, 16, 1)   # group must be 64
    assert moe.lib.moe_ctx_create(C.byref(bad), 0, C.byref(h)) == moe.MOE_ERR_ARG
    bad = moe.moe_dims(2816, 128, 8, 704, 2112, 64, 4, 1)    # fewer slots than top_k
    assert moe.lib.moe_ctx_create(C.byref(bad), 0, C.byref(h)) == moe.MOE_ERR_ARG
    bad = moe.moe_dims(16384, 128, 8, 704, 2112, 64, 16, 1)  # wider than the batched kernels stage
    assert moe.lib.moe_ctx_create(C.byref(bad), 0, C.byref(h)) == moe.MOE_ERR_ARG
    bad = moe.moe_dims(2816, 132, 8, 704, 2112, 64, 16, 1)   # experts not a multiple of the router cluster
    assert moe.lib.moe_ctx_create(C.byref(bad), 0, C.byref(h)) == moe.MOE_ERR_ARG
    assert moe.lib.moe_ctx_create(C.byref(bad), 0, None) == moe.MOE_ERR_ARG


def test_header_documents_every_entry_point():
    src = open(moe.HEADER).read()
    for name in moe.declared_symbols():
        # each declaration is preceded by a comment block
        m = re.search(r"\*/\s*(?:[\w\s\*]+?)\b" + name + r"\s*\(", src)
        assert m, name


def test_attn_host_side_checks_without_a_gpu():
    """Workspace sizing is host arithmetic; argument checks of the decode
    attention entry point answer before any CUDA call."""
    # ticket block + per (query head, part) an (m, l) pair and head_dim partial sums
    assert moe.attn_workspace_bytes(16, 256) == 256 + 16 * 64 * 8 + 16 * 64 * 256 * 4
    assert moe.attn_workspace_bytes(0, 256) == 0
    L = moe.lib
    ok = dict(q=16, k=16, v=16, hq=4, hkv=2, hd=64, cap=8, n=4, scale=0.1, o=16, ws=16, wsb=1 << 20)

    def call(**kw):
        a = {**ok, **kw}
        return L.moe_attn_decode(a["q"], a["k"], a["v"], a["hq"], a["hkv"], a["hd"], a["cap"], a["n"], a["scale"],
                                 a["o"], a["ws"], a["wsb"], None)

    # fake (aligned, never dereferenced) addresses: each case fails a check first
    assert call(q=None) == moe.MOE_ERR_ARG
    assert call(n=0) == moe.MOE_ERR_ARG
    assert call(cap=0) == moe.MOE_ERR_ARG
    assert call(hd=96) == moe.MOE_ERR_ARG
    assert call(hq=6, hkv=4) == moe.MOE_ERR_ARG
    assert call(hq=32, hkv=2) == moe.MOE_ERR_ARG
    assert call(hd=512, hq=8, hkv=2) == moe.MOE_ERR_ARG   # group 4 at width 512: too many registers
    assert call(scale=-1.0) == moe.MOE_ERR_ARG
    assert call(q=18) == moe.MOE_ERR_ARG                  # not 16-byte aligned
    assert call(wsb=100) == moe.MOE_ERR_ARG
