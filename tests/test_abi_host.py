"""Host-side checks of the C ABI: the library loads, exports every symbol the header
declares, and rejects bad arguments before anything reaches a GPU.  None of these
calls launches a kernel, so they run without a GPU."""
import ctypes
import os
import re

import pytest

import decode_attention_quant_b200 as dq
from decode_attention_quant_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "wushkv.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wushkv_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    lib = dq.library()
    declared = _declared_symbols()
    assert declared == sorted(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_strerror():
    lib = dq.library()
    assert lib.wushkv_version().startswith(b"wushkv")
    for code in (0, -1, -2, -3, -4, -5, 7):
        assert isinstance(_lib.strerror(code), str)


def _desc(**kw):
    qp = _lib.QuantParams(kw.pop("kind", 0), kw.pop("bits", 2), kw.pop("alpha", 1.99), kw.pop("rlo", 2),
                          kw.pop("rhi", 125))
    fields = dict(k_codes=0x10000, v_codes=0x20000, k_meta=0x30000, v_meta=0x40000, batch=2,
                  num_kv_heads=2, capacity=256, head_dim=128)
    fields.update(kw)
    return _lib.CacheDesc(fields["k_codes"], fields["v_codes"], fields["k_meta"], fields["v_meta"],
                          fields["batch"], fields["num_kv_heads"], fields["capacity"], fields["head_dim"], qp)


BAD_CACHES = [
    (dict(head_dim=64), _lib.ERR_UNSUPPORTED),
    (dict(bits=1), _lib.ERR_UNSUPPORTED),
    (dict(bits=5), _lib.ERR_UNSUPPORTED),
    (dict(kind=7), _lib.ERR_UNSUPPORTED),
    (dict(batch=0), _lib.ERR_INVALID),
    (dict(capacity=0), _lib.ERR_INVALID),
    (dict(alpha=0.0), _lib.ERR_INVALID),
    (dict(alpha=float("nan")), _lib.ERR_INVALID),
    (dict(kind=1, rlo=5, rhi=4), _lib.ERR_INVALID),
    (dict(kind=1, rlo=10, rhi=120), _lib.ERR_UNSUPPORTED),
    (dict(k_codes=0), _lib.ERR_INVALID),
    (dict(v_codes=0x20008), _lib.ERR_MISALIGNED),
    (dict(k_meta=0x30002), _lib.ERR_MISALIGNED),
]


@pytest.mark.parametrize("kw,code", BAD_CACHES)
def test_append_rejects_bad_cache(kw, code):
    lib = dq.library()
    d = _desc(**kw)
    rc = lib.wushkv_quantize_append(ctypes.byref(d), 0x50000, 0x60000, 0, 4, 0x70000, None, None, None)
    assert rc == code
    if "alpha" not in kw:        # the clip multiplier only matters when quantizing
        assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 0) == 0
    else:
        assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 0) > 0


def test_append_rejects_bad_arguments():
    lib = dq.library()
    d = _desc()
    call = lib.wushkv_quantize_append
    assert call(None, 0x50000, 0x60000, 0, 4, 0x70000, None, None, None) == _lib.ERR_INVALID
    assert call(ctypes.byref(d), 0x50000, 0x60000, 9, 4, 0x70000, None, None, None) == _lib.ERR_UNSUPPORTED
    assert call(ctypes.byref(d), 0x50000, 0x60000, 0, 0, 0x70000, None, None, None) == _lib.ERR_INVALID
    assert call(ctypes.byref(d), None, 0x60000, 0, 4, 0x70000, None, None, None) == _lib.ERR_INVALID
    assert call(ctypes.byref(d), 0x50000, 0x60000, 0, 4, None, None, None, None) == _lib.ERR_INVALID
    assert call(ctypes.byref(d), 0x50004, 0x60000, 0, 4, 0x70000, None, None, None) == _lib.ERR_MISALIGNED
    assert call(ctypes.byref(d), 0x50000, 0x60000, 0, 4, 0x70002, None, None, None) == _lib.ERR_MISALIGNED
    assert call(ctypes.byref(d), 0x50000, 0x60000, 0, 4, 0x70000, 0x80004, None, None) == _lib.ERR_MISALIGNED


def test_transform_query_rejects_bad_arguments():
    f = dq.library().wushkv_transform_query
    assert f(0x1000, 3, 2, 32, 8, 0x2000, 0x3000, None) == _lib.ERR_UNSUPPORTED
    assert f(0x1000, 0, 2, 30, 8, 0x2000, 0x3000, None) == _lib.ERR_INVALID
    assert f(0x1000, 0, 2, 96, 4, 0x2000, 0x3000, None) == _lib.ERR_UNSUPPORTED   # g = 24
    assert f(0x1000, 0, 0, 32, 8, 0x2000, 0x3000, None) == _lib.ERR_INVALID
    assert f(0x1000, 0, 2, 32, 8, None, 0x3000, None) == _lib.ERR_INVALID
    assert f(0x1000, 0, 2, 32, 8, 0x2000, 0x1000, None) == _lib.ERR_INVALID       # aliasing
    assert f(0x1004, 0, 2, 32, 8, 0x2000, 0x3000, None) == _lib.ERR_MISALIGNED


def test_decode_rejects_bad_arguments():
    lib = dq.library()
    d = _desc()
    need = lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 0)
    assert need > 0
    assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 3) == 2 * 4 * 3 * 132 * 4
    assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 3, 0) == 0
    f = lib.wushkv_decode_attention
    ok = (ctypes.byref(d), 0x1000, 4, 0x2000, 0.1, 0x3000, 0x4000, need, 0, None, None)

    def call(**kw):
        args = list(ok)
        names = ["c", "q", "hq", "ctx", "scale", "out", "ws", "wsb", "ns", "st", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)

    assert call(ws=0x4000, wsb=need - 1) == _lib.ERR_WORKSPACE
    assert call(q=None) == _lib.ERR_INVALID
    assert call(hq=5) == _lib.ERR_INVALID
    assert call(hq=6) == _lib.ERR_UNSUPPORTED
    assert call(ns=-1) == _lib.ERR_INVALID
    assert call(scale=float("inf")) == _lib.ERR_INVALID
    assert call(out=0x3004) == _lib.ERR_MISALIGNED
    assert call(ctx=0x2002) == _lib.ERR_MISALIGNED
    assert call(st=0x5002) == _lib.ERR_MISALIGNED


PAGED_BAD = [
    (dict(block_table=0x50000, pages_per_seq=4, page_size=48, num_pages=16, capacity=192), _lib.ERR_INVALID),
    (dict(block_table=0x50000, pages_per_seq=4, page_size=8, num_pages=16, capacity=32), _lib.ERR_INVALID),
    (dict(block_table=0x50000, pages_per_seq=4, page_size=64, num_pages=16, capacity=200), _lib.ERR_INVALID),
    (dict(block_table=0x50000, pages_per_seq=0, page_size=64, num_pages=16, capacity=0), _lib.ERR_INVALID),
    (dict(block_table=0x50000, pages_per_seq=4, page_size=64, num_pages=0, capacity=256), _lib.ERR_INVALID),
    (dict(block_table=0x50002, pages_per_seq=4, page_size=64, num_pages=16, capacity=256), _lib.ERR_MISALIGNED),
]


@pytest.mark.parametrize("fields,code", PAGED_BAD)
def test_paged_layout_checks(fields, code):
    """Paged caches: page size a power of two in [16, 4096], capacity = pages x page size,
    a non-empty pool and an aligned block table; rejected before any launch."""
    d = _desc(capacity=fields.pop("capacity"))
    for k, v in fields.items():
        setattr(d, k, v)
    lib = dq.library()
    assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 1) == 0
    vp = ctypes.c_void_p
    rc = lib.wushkv_decode_attention(ctypes.byref(d), vp(0x60000), 4, vp(0x70000), 0.1, vp(0x80000),
                                     vp(0x90000), 1 << 20, 1, vp(0), vp(0))
    assert rc == code


def test_paged_layout_accepted():
    d = _desc(capacity=256)
    d.block_table, d.pages_per_seq, d.page_size, d.num_pages = 0x50000, 4, 64, 16
    assert dq.library().wushkv_decode_workspace_bytes(ctypes.byref(d), 4, 1) > 0


def test_chunk_workspace_and_argument_checks():
    lib = dq.library()
    d = _desc()
    # layout: one partial (m, l, pad, pad, o[128]) per (sequence, chunk query, query head, split)
    def floats(hq, n_q, splits):
        return 2 * n_q * hq * splits * 132
    assert lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 4, 16, 3) == 4 * floats(4, 16, 3) == 202752
    assert lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 4, 3, 3) == 4 * floats(4, 3, 3) == 38016
    assert lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 4, 0, 0) == 0
    assert lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 4, 17, 0) == 0
    assert lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 6, 4, 0) == 0
    need = lib.wushkv_chunk_workspace_bytes(ctypes.byref(d), 4, 16, 0)
    assert need > 0
    f = lib.wushkv_chunk_attention
    ok = (ctypes.byref(d), 0x1000, 16, 4, 0x2000, 0.1, 0x3000, 0x4000, need, 0, None, None)

    def call(**kw):
        args = list(ok)
        names = ["c", "q", "nq", "hq", "ctx", "scale", "out", "ws", "wsb", "ns", "st", "stream"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return f(*args)

    assert call(wsb=need - 1) == _lib.ERR_WORKSPACE
    assert call(nq=0) == _lib.ERR_INVALID
    assert call(nq=17) == _lib.ERR_INVALID
    assert call(q=None) == _lib.ERR_INVALID
    assert call(out=0x1000) == _lib.ERR_INVALID
    assert call(hq=6) == _lib.ERR_UNSUPPORTED
    assert call(ns=-1) == _lib.ERR_INVALID
    assert call(scale=float("nan")) == _lib.ERR_INVALID
    assert call(q=0x1008) == _lib.ERR_MISALIGNED
    assert call(ws=0x4008) == _lib.ERR_MISALIGNED
    assert call(ctx=0x2002) == _lib.ERR_MISALIGNED


def test_append_rope_argument_checks():
    lib = dq.library()
    d = _desc()                                          # batch 2, Hkv 2, capacity 256
    f = lib.wushkv_quantize_append_rope
    ok = (ctypes.byref(d), 0x50000, 0x60000, 0, 4, 0x70000, None, 0x80000, 256, None, None)

    def call(**kw):
        args = list(ok)
        names = ["c", "k", "v", "dt", "n", "sp", "tk", "tab", "rows", "st", "stream"]
        for key, val in kw.items():
            args[names.index(key)] = val
        return f(*args)

    assert call(tab=None) == _lib.ERR_INVALID
    assert call(rows=255) == _lib.ERR_INVALID            # the table must cover the capacity
    assert call(tab=0x80008) == _lib.ERR_MISALIGNED
    assert call(n=33) == _lib.ERR_UNSUPPORTED            # 66 token rows: not a decode-step append
    assert call(dt=1) == _lib.ERR_UNSUPPORTED            # fp32 keys
    assert call(dt=7) == _lib.ERR_UNSUPPORTED
    assert call(n=0) == _lib.ERR_INVALID


def test_append_structured_argument_checks():
    lib = dq.library()
    d = _desc()
    f = lib.wushkv_quantize_append_structured
    ok = (ctypes.byref(d), 0x50000, 0x60000, 0, 4, 0x70000, 2, 32, 0x80000, None, None)

    def call(**kw):
        args = list(ok)
        names = ["c", "k", "v", "dt", "n", "sp", "kind", "block", "data", "st", "stream"]
        for key, val in kw.items():
            args[names.index(key)] = val
        return f(*args)

    assert call(kind=9) == _lib.ERR_UNSUPPORTED
    assert call(block=8) == _lib.ERR_UNSUPPORTED
    assert call(block=128) == _lib.ERR_UNSUPPORTED
    assert call(data=None) == _lib.ERR_INVALID
    assert call(data=0x80004) == _lib.ERR_MISALIGNED
    assert call(n=0) == _lib.ERR_INVALID
    assert call(kind=3, dt=1) == _lib.ERR_UNSUPPORTED     # fp32 keys
    assert call(kind=1, data=None) == _lib.ERR_INVALID    # dense needs its matrix
    assert call(kind=1, dt=7) == _lib.ERR_UNSUPPORTED     # dense forwards to the plain append's checks


def test_transform_query_structured_argument_checks():
    lib = dq.library()
    f = lib.wushkv_transform_query_structured
    ok = (0x50000, 0, 2, 32, 8, 2, 32, 0x80000, 0x90000, None)

    def call(**kw):
        args = list(ok)
        names = ["q", "dt", "b", "hq", "hkv", "kind", "block", "data", "out", "stream"]
        for key, val in kw.items():
            args[names.index(key)] = val
        return f(*args)

    assert call(kind=9) == _lib.ERR_UNSUPPORTED
    assert call(block=8) == _lib.ERR_UNSUPPORTED
    assert call(dt=5) == _lib.ERR_UNSUPPORTED
    assert call(hq=20) == _lib.ERR_INVALID              # not a multiple of the KV heads
    assert call(hq=24) == _lib.ERR_UNSUPPORTED          # group size 3
    assert call(b=0) == _lib.ERR_INVALID
    assert call(data=None) == _lib.ERR_INVALID
    assert call(out=0x50000) == _lib.ERR_INVALID        # output may not alias q
    assert call(data=0x80004) == _lib.ERR_MISALIGNED
    assert call(kind=3, q=0x50008) == _lib.ERR_MISALIGNED
    assert call(kind=1, data=None) == _lib.ERR_INVALID  # dense forwards to wushkv_transform_query
