"""The allocation-free decode entry (wushkv_decode_attention_noalloc): same results
as wushkv_decode_attention with a caller workspace, through the C ABI, on two calls
in a row whose second call must not see the first call's partials; and the host-side
rejection of calls whose partials do not fit the fixed scratch array.

The file name sorts last so that the GPU case also runs after every other test has
used the device; it passes alone in a fresh process too.
"""
import ctypes
import math

import pytest
import torch

import decode_attention_quant_b200 as dq
from decode_attention_quant_b200 import _lib
from synth import gen

TAU = 1.0 / math.sqrt(128)


def _fake_desc(batch, num_kv_heads, capacity):
    qp = _lib.QuantParams(1, 2, 0.0, 2, 125)
    return _lib.CacheDesc(0x10000, 0x20000, 0x30000, 0x40000, batch, num_kv_heads, capacity, 128, qp)


def test_rejects_oversized_and_invalid_without_launching():
    lib = dq.library()
    vp = ctypes.c_void_p
    # 2048 sequences x 32 query heads x 1 split x 528 bytes > 8 MiB of scratch
    d = _fake_desc(2048, 8, 256)
    assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 32, 1) > _lib.DECODE_STATIC_SCRATCH_BYTES
    rc = lib.wushkv_decode_attention_noalloc(ctypes.byref(d), vp(0x50000), 32, vp(0x60000), TAU, vp(0x70000),
                                             1, vp(0), vp(0))
    assert rc == _lib.ERR_WORKSPACE
    # invalid arguments report the regular entry's codes
    assert lib.wushkv_decode_attention_noalloc(None, vp(0x50000), 32, vp(0x60000), TAU, vp(0x70000), 1,
                                               vp(0), vp(0)) == _lib.ERR_INVALID
    d = _fake_desc(2, 8, 256)
    assert lib.wushkv_decode_attention_noalloc(ctypes.byref(d), vp(0x50000), 24, vp(0x60000), TAU, vp(0x70000),
                                               1, vp(0), vp(0)) == _lib.ERR_UNSUPPORTED
    assert lib.wushkv_decode_attention_noalloc(ctypes.byref(d), vp(0x50000), 32, vp(0x60000), TAU, vp(0x70000),
                                               -1, vp(0), vp(0)) == _lib.ERR_INVALID
    # a split count out of range is invalid whatever the scratch it would need
    d = _fake_desc(2048, 8, 256)
    assert lib.wushkv_decode_workspace_bytes(ctypes.byref(d), 32, 5000) == 0
    assert lib.wushkv_decode_attention_noalloc(ctypes.byref(d), vp(0x50000), 32, vp(0x60000), TAU, vp(0x70000),
                                               5000, vp(0), vp(0)) == _lib.ERR_INVALID


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls():
    kind, bits, batch, hq, hkv, cap = 1, 2, 4, 32, 8, 4096
    c = gen.random_cache(batch, hkv, cap, kind, bits, seed=21, device="cuda")
    cache = dq.PackedCache(batch, hkv, cap, kind, bits, tensors=c)
    g = torch.Generator(device="cuda").manual_seed(5)
    q1 = torch.randn(batch, hq, 128, generator=g, device="cuda") * 2.0
    q2 = torch.randn(batch, hq, 128, generator=g, device="cuda") * 2.0
    ctx1 = torch.tensor([4096, 3000, 129, 4001], dtype=torch.int32, device="cuda")
    ctx2 = torch.tensor([17, 0, 4096, 1500], dtype=torch.int32, device="cuda")
    assert dq.decode_workspace_bytes(cache, hq) <= _lib.DECODE_STATIC_SCRATCH_BYTES

    got1 = dq.decode_attention_noalloc(cache, q1, ctx1, TAU)
    got2 = dq.decode_attention_noalloc(cache, q2, ctx2, TAU)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got3 = dq.decode_attention_noalloc(cache, q1, ctx1, TAU, num_splits=3, status=st)
    ref1 = dq.decode_attention(cache, q1, ctx1, TAU)
    ref2 = dq.decode_attention(cache, q2, ctx2, TAU)
    ref3 = dq.decode_attention(cache, q1, ctx1, TAU, num_splits=3)
    torch.cuda.synchronize()
    for got, ref in ((got1, ref1), (got2, ref2), (got3, ref3)):
        assert torch.isfinite(got).all()
        assert torch.allclose(got, ref, rtol=0, atol=5e-5), (got - ref).abs().max()
    assert torch.all(got2[1] == 0)                           # ctx_len 0 -> zero rows, not stale partials
    assert st.item() == 0
