"""GPU parity of wushkv_quantize_append_rope (RoPE fused in front of the key transform,
decode-step appends) against the oracle's quantize_append_rope, on the same pre-RoPE
bf16 keys and the same fp32 cos/sin table.

Bar, as for the other end-to-end appends: value codes and meta bit-exact; key meta may
differ by one fp16 ulp only within 1e-4 * Delta of an fp16 midpoint; key codes by +-1
only within 1e-4 * Delta of a decision threshold (the GPU rotates and transforms in
fp32, the oracle in fp64).
"""
import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QUEST_ALPHA, QWEN8B_DECODE
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
CASES = [(0, 2), (0, 3), (0, 4), (1, 2), (1, 3), (1, 4)]


def _alpha(kind, bits):
    return QUEST_ALPHA[bits] if kind == orc.QUEST_INT else 0.0


def _run(k_pre, v, tk, table, kind, bits, start, cap):
    bsz, n, hkv, _ = k_pre.shape
    alpha = _alpha(kind, bits)
    oc = orc.empty_cache(bsz, hkv, cap, kind, bits)
    ost = orc.quantize_append_rope(oc, gu.to_numpy64(k_pre), gu.to_numpy64(v), start, table.numpy(), kind, bits,
                                   alpha, 2, 125, tk=None if tk is None else tk.numpy().astype(np.float64))
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, alpha)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append_rope(cache, k_pre.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32, device="cuda"),
                            table.cuda(), None if tk is None else tk.cuda(), status=st)
    torch.cuda.synchronize()
    return oc, ost, gu.cache_to_numpy(cache), int(st.item())


def _oracle_x(k_pre, tk, table, start):
    """The oracle's rotated and transformed keys [B, n, Hkv, 128] (R19, R1)."""
    k = gu.to_numpy64(k_pre)
    tab = table.numpy().astype(np.float64)
    rot = np.empty_like(k)
    for b in range(k.shape[0]):
        for t in range(k.shape[1]):
            p = start[b] + t
            rot[b, t] = orc.apply_rope(k[b, t], tab[p, :64], tab[p, 64:])
    return rot if tk is None else orc.transform_keys(rot, tk.numpy().astype(np.float64))


@pytest.mark.parametrize("kind,bits", CASES)
@pytest.mark.parametrize("bsz,n", [(16, 1), (4, 16)])
def test_rope_append_end_to_end(kind, bits, bsz, n):
    w = QWEN8B_DECODE
    hkv, cap = 2, 4096
    start = [(977 * b) % 4000 for b in range(bsz)]            # positions spread over the table
    tk = torch.from_numpy(gen.transforms(w)[0][:hkv].copy())
    table = gen.rope_table(cap, w.rope_theta)
    k = gen.keys(w, 0, bsz, start, n, rope=False)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    oc, ost, gc, gst = _run(k, v, tk, table, kind, bits, start, cap)
    assert ost == 0 and gst == 0
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    np.testing.assert_array_equal(oc["v_meta"], gc["v_meta"])
    flips, diffs, near = gu.check_key_rows(oc, gc, _oracle_x(k, tk, table, start), kind, bits, start,
                                           _alpha(kind, bits))
    print(f"kind={kind} bits={bits} B={bsz} n={n}: key meta flips {flips}, key code diffs {diffs} "
          f"(values within 1e-4*Delta of a boundary: {near})")


@pytest.mark.parametrize("kind,bits", [(0, 2), (1, 4)])
def test_rope_append_without_transform(kind, bits):
    w = QWEN8B_DECODE
    bsz, n, hkv, cap = 8, 2, 2, 64
    start = [5 * b for b in range(bsz)]
    table = gen.rope_table(cap, w.rope_theta)
    k = gen.keys(w, 0, bsz, start, n, rope=False)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    oc, ost, gc, gst = _run(k, v, None, table, kind, bits, start, cap)
    assert ost == 0 and gst == 0
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    gu.check_key_rows(oc, gc, _oracle_x(k, None, table, start), kind, bits, start, _alpha(kind, bits))


def test_rope_identity_table_equals_plain_append():
    """cos = 1, sin = 0 leaves every key as it is: the fused call writes exactly what the
    plain append of the same keys writes."""
    w = QWEN8B_DECODE
    bsz, n, hkv, cap = 16, 1, 8, 32
    start = [b for b in range(bsz)]
    tk = torch.from_numpy(gen.transforms(w)[0].copy()).cuda()
    k = gen.keys(w, 0, bsz, start, n).cuda()
    v = gen.values(w, 0, bsz, start, n).cuda()
    ident = torch.cat([torch.ones(cap, 64), torch.zeros(cap, 64)], dim=1).cuda()
    sp = torch.tensor(start, dtype=torch.int32, device="cuda")
    a = dq.PackedCache(bsz, hkv, cap, 1, 2)
    b = dq.PackedCache(bsz, hkv, cap, 1, 2)
    dq.quantize_append_rope(a, k, v, sp, ident, tk)
    dq.quantize_append(b, k, v, sp, tk)
    for x, y in zip(a.tensors().values(), b.tensors().values()):
        assert torch.equal(x, y)


def test_rope_append_capacity_status():
    w = QWEN8B_DECODE
    bsz, n, hkv, cap = 3, 2, 1, 10
    start = [2, 9, 0]                                          # sequence 1 writes positions 9, 10 (= cap)
    table = gen.rope_table(cap, w.rope_theta)
    tk = torch.from_numpy(gen.transforms(w)[0][:hkv].copy())
    k = gen.keys(w, 0, bsz, start, n, rope=False)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    oc, ost, gc, gst = _run(k, v, tk, table, 1, 2, start, cap)
    assert ost & orc.STATUS_CAPACITY and gst & dq.STATUS_CAPACITY
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    np.testing.assert_array_equal(oc["v_meta"], gc["v_meta"])
