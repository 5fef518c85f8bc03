"""GPU parity of wushkv_transform_query and wushkv_decode_attention against the CPU
oracle, on the same packed codes (built by the oracle's append or drawn at random).

Bar: attention max-abs error <= 2e-3 and relative L2 <= 1e-2 against the fp64
oracle; transformed queries within 1e-5 relative (fp32 arithmetic over 128 terms).
"""
import math

import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QUEST_ALPHA, QWEN8B_DECODE, TINY
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
TAU = 1.0 / math.sqrt(128)
MAX_ABS, REL_L2 = 2e-3, 1e-2


def _oracle_cache(w, bsz, hkv, n, cap, kind, bits, tk):
    k = gen.keys(w, 0, bsz, 0, n)[:, :, :hkv]
    v = gen.values(w, 0, bsz, 0, n)[:, :, :hkv]
    oc = orc.empty_cache(bsz, hkv, cap, kind, bits)
    alpha = QUEST_ALPHA[bits] if kind == 0 else 0.0
    assert orc.quantize_append(oc, gu.to_numpy64(k), gu.to_numpy64(v), [0] * bsz, kind, bits, alpha, 2, 125,
                               tk=tk[:hkv].astype(np.float64)) == 0
    return oc


def test_transform_query_matches_oracle():
    w = QWEN8B_DECODE
    _, tinv = gen.transforms(w)
    q = gen.queries(w)                                  # bf16 [16, 32, 128]
    got = dq.transform_query(q.cuda(), torch.from_numpy(tinv).cuda(), w.num_kv_heads)
    ref = orc.transform_query(gu.to_numpy64(q), tinv.astype(np.float64), w.num_kv_heads)
    err = np.abs(got.cpu().numpy() - ref) / (np.abs(ref).max(axis=-1, keepdims=True) + 1e-30)
    assert err.max() < 1e-5, err.max()
    got32 = dq.transform_query(q.float().cuda(), torch.from_numpy(tinv).cuda(), w.num_kv_heads)
    assert torch.allclose(got, got32, rtol=0, atol=0)


@pytest.mark.parametrize("kind,bits,hq,hkv,ctx", [
    (0, 2, 4, 1, [256]),                   # the tiny single-layer workload
    (1, 2, 8, 2, [300, 77]),
    (0, 3, 8, 2, [129, 5]),
    (0, 4, 16, 2, [200, 1]),
    (1, 4, 4, 4, [128, 260]),
])
def test_decode_matches_oracle_on_oracle_cache(kind, bits, hq, hkv, ctx):
    w = TINY if hq == 4 and hkv == 1 else QWEN8B_DECODE
    bsz, cap = len(ctx), max(ctx) + 16
    tk, tinv = gen.transforms(QWEN8B_DECODE)
    oc = _oracle_cache(w, bsz, hkv, max(ctx), cap, kind, bits, tk)
    q = gen.queries(QWEN8B_DECODE)[:bsz, :hq]
    qt_ref = orc.transform_query(gu.to_numpy64(q), tinv[:hkv].astype(np.float64), hkv)
    qt32 = torch.from_numpy(qt_ref.astype(np.float32))
    ref = orc.decode_attention(oc, qt32.numpy().astype(np.float64), ctx, TAU, kind, bits, hkv)
    cache = gu.cache_to_gpu(oc, kind, bits)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    got = dq.decode_attention(cache, qt32.cuda(), ctx_t, TAU).cpu().numpy()
    ma, rl = gu.attention_errors(got, ref)
    print(f"kind={kind} bits={bits} g={hq // hkv}: max-abs {ma:.3e} rel-L2 {rl:.3e}")
    assert ma <= MAX_ABS and rl <= REL_L2
    # end to end through the GPU query transform
    qt_gpu = dq.transform_query(q.contiguous().cuda(), torch.from_numpy(tinv[:hkv].copy()).cuda(), hkv)
    got2 = dq.decode_attention(cache, qt_gpu, ctx_t, TAU).cpu().numpy()
    ref2 = orc.decode_attention(oc, qt_ref, ctx, TAU, kind, bits, hkv)
    ma2, rl2 = gu.attention_errors(got2, ref2)
    assert ma2 <= MAX_ABS and rl2 <= REL_L2


def test_split_count_invariance_and_edges():
    kind, bits, hq, hkv = 1, 2, 8, 2
    bsz, cap = 3, 1100
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=5, device="cpu")
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors={k: v.cuda() for k, v in c.items()})
    q = torch.randn(bsz, hq, 128, generator=torch.Generator().manual_seed(3)).cuda()
    ctx = torch.tensor([1100, 0, 513], dtype=torch.int32, device="cuda")
    outs = [dq.decode_attention(cache, q, ctx, TAU, num_splits=s) for s in (1, 0, 3, 7, 9)]
    # splits change only where the 16-bit probability limbs are rounded (per tile scale)
    for o in outs[1:]:
        assert torch.allclose(o, outs[0], rtol=0, atol=5e-5), (o - outs[0]).abs().max()
    assert torch.all(outs[0][1] == 0)                 # ctx_len 0 -> zero rows
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    over = dq.decode_attention(cache, q, torch.tensor([5000, 0, 513], dtype=torch.int32, device="cuda"),
                               TAU, status=st)
    torch.cuda.synchronize()
    assert st.item() & dq.STATUS_CTX_OVERFLOW
    assert torch.allclose(over, outs[0], rtol=0, atol=5e-5)


@pytest.mark.parametrize("kind,bits,batch,hq,hkv,ctx", [
    (1, 2, 16, 32, 8, 32768),            # Qwen3-8B-shaped decode layer, affine 2-bit
    (0, 3, 16, 32, 8, 32768),            # QuEST 3-bit sweep point
    (1, 2, 4, 32, 8, 131072),            # long-context split-K
    (0, 2, 32, 64, 8, 8192),             # Qwen3-32B-shaped layer, QuEST 2-bit
])
def test_decode_full_size_sampled(kind, bits, batch, hq, hkv, ctx):
    """Full-size random caches; the oracle checks a deterministic sample of (sequence, KV head) pairs."""
    c = gen.random_cache(batch, hkv, ctx, kind, bits, seed=ctx + batch, device="cuda")
    cache = dq.PackedCache(batch, hkv, ctx, kind, bits, tensors=c)
    g = torch.Generator(device="cuda").manual_seed(11)
    q = torch.randn(batch, hq, 128, generator=g, device="cuda") * 2.0
    ctx_t = torch.full((batch,), ctx, dtype=torch.int32, device="cuda")
    ctx_t[-1] = ctx - 77                                       # ragged tail on one sequence
    out = dq.decode_attention(cache, q, ctx_t, TAU).cpu().numpy()
    gsz = hq // hkv
    qn = q.cpu().numpy().astype(np.float64)
    ctx_h = ctx_t.cpu().numpy()
    for (b, kv) in [(0, 0), (batch - 1, hkv - 1), (batch // 2, 3 % hkv)]:
        n = int(ctx_h[b])
        kc = c["k_codes"][b, kv, :n].cpu().numpy()
        vc = c["v_codes"][b, kv, :n].cpu().numpy()
        km = c["k_meta"][b, kv, :n].cpu().numpy().view(np.uint16)
        vm = c["v_meta"][b, kv, :n].cpu().numpy().view(np.uint16)
        ref = orc.decode_attention_pair(kc, km, vc, vm, qn[b, kv * gsz:(kv + 1) * gsz], TAU, kind, bits)
        ma, rl = gu.attention_errors(out[b, kv * gsz:(kv + 1) * gsz], ref)
        assert ma <= MAX_ABS and rl <= REL_L2, (b, kv, ma, rl)


@pytest.mark.parametrize("kind,bits", [(1, 2), (0, 2), (0, 3), (1, 4)])
def test_flat_attention_over_maximal_value_codes(kind, bits):
    """Equal scores over whole tiles and every value code at its maximum: the largest
    value sums a tile can produce (each limb column near 255 x 240 x 256), so any int32
    overflow in combining them would show.  The output is the dequantized top code."""
    bsz, hkv, hq, ctx = 2, 2, 8, 1024
    c = gen.random_cache(bsz, hkv, ctx, kind, bits, seed=7, device="cpu")
    c["k_codes"][:] = c["k_codes"][:, :, :1].clone()          # one key row repeated: equal scores
    c["k_meta"][:] = c["k_meta"][:, :, :1].clone()
    c["v_codes"][:] = 0xFF                                     # every value code = 2^b - 1
    c["v_meta"][:] = c["v_meta"][:, :, :1].clone()             # equal value scales: e * scale at the cap
    cache = dq.PackedCache(bsz, hkv, ctx, kind, bits, tensors={k: v.cuda() for k, v in c.items()})
    q = torch.randn(bsz, hq, 128, generator=torch.Generator().manual_seed(4)) * 2.0
    ctx_t = torch.full((bsz,), ctx, dtype=torch.int32, device="cuda")
    for ns in (0, 1):                                          # automatic split count, and one split
        out = dq.decode_attention(cache, q.cuda(), ctx_t, TAU, num_splits=ns).cpu().numpy()
        gsz = hq // hkv
        for b in range(bsz):
            for kv in range(hkv):
                km = c["k_meta"][b, kv].numpy().view(np.uint16)
                vm = c["v_meta"][b, kv].numpy().view(np.uint16)
                ref = orc.decode_attention_pair(c["k_codes"][b, kv].numpy(), km, c["v_codes"][b, kv].numpy(), vm,
                                                q[b, kv * gsz:(kv + 1) * gsz].numpy().astype(np.float64), TAU,
                                                kind, bits)
                ma, rl = gu.attention_errors(out[b, kv * gsz:(kv + 1) * gsz], ref)
                assert ma <= MAX_ABS and rl <= REL_L2, (ns, b, kv, ma, rl)
