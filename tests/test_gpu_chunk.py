"""GPU parity of wushkv_chunk_attention (causal attention of an n_q-query chunk over
the packed cache) against the CPU oracle, on the same packed codes.

Bar: attention max-abs error <= 2e-3 and relative L2 <= 1e-2 against the fp64 oracle,
as for decode.  Query i of a chunk sits at position ctx - n_q + i; queries before
position 0 give zero rows.
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


def _chunk_queries(bsz, n_q, hq, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(bsz, n_q, hq, 128, generator=g) * 1.5).contiguous()


@pytest.mark.parametrize("kind,bits,hq,hkv,n_q,ctx", [
    (0, 2, 4, 1, 16, [256]),               # tiny workload shape, one 16-token chunk at the end
    (1, 2, 8, 2, 16, [300, 20]),           # g = 4: 64 folded rows in one 128-row block
    (0, 3, 16, 2, 16, [129, 7]),           # g = 8: one full row block; sequence 1 shorter than the chunk
    (0, 4, 2, 2, 5, [260, 16]),            # g = 1, n_q = 5: 5 rows of a block
    (1, 4, 32, 2, 16, [1000, 513]),        # g = 16: 256 folded rows, two row blocks
    (1, 3, 8, 2, 1, [77, 300]),            # n_q = 1: a decode query
])
def test_chunk_matches_oracle(kind, bits, hq, hkv, n_q, ctx):
    w = TINY if hkv == 1 else QWEN8B_DECODE
    bsz, cap = len(ctx), max(ctx) + 16
    tk, _ = gen.transforms(QWEN8B_DECODE)
    oc = _oracle_cache(w, bsz, hkv, max(ctx), cap, kind, bits, tk)
    q = _chunk_queries(bsz, n_q, hq, seed=hq + n_q)
    ref = orc.chunk_attention(oc, q.numpy().astype(np.float64), ctx, TAU, kind, bits, hkv)
    cache = gu.cache_to_gpu(oc, kind, bits)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = dq.chunk_attention(cache, q.cuda(), ctx_t, TAU, status=st).cpu().numpy()
    torch.cuda.synchronize()
    assert st.item() == 0
    ma, rl = gu.attention_errors(got, ref)
    print(f"kind={kind} bits={bits} g={hq // hkv} n_q={n_q}: max-abs {ma:.3e} rel-L2 {rl:.3e}")
    assert ma <= MAX_ABS and rl <= REL_L2
    for b, n in enumerate(ctx):                      # queries before position 0: zero rows
        for i in range(n_q):
            if n - n_q + i < 0:
                assert np.all(got[b, i] == 0), (b, i)


@pytest.mark.parametrize("kind,bits,hq,hkv", [(0, 2, 8, 2), (1, 4, 16, 2), (0, 3, 4, 1)])
def test_chunk_multi_tile_ctas(kind, bits, hq, hkv):
    """One CTA walks many 128-position tiles (num_splits 1 and 2): double-buffered
    operands, O accumulated across tiles, and the running reference moving for some rows
    of a warp but not for others (queries scaled up so that tile maxima spread by more
    than 2^8)."""
    n_q, bsz, cap = 16, 2, 1000
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=31 + bits, device="cpu")
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors={k: v.cuda() for k, v in c.items()})
    q = (_chunk_queries(bsz, n_q, hq, seed=40 + hq) * 4.0).contiguous()
    ctx = [1000, 611]
    cn = {name: t.numpy() for name, t in c.items()}
    cn["k_meta"] = cn["k_meta"].view(np.uint16)
    cn["v_meta"] = cn["v_meta"].view(np.uint16)
    ref = orc.chunk_attention(cn, q.numpy().astype(np.float64), ctx, TAU, kind, bits, hkv)
    ctx_t = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    for s in (1, 2):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = dq.chunk_attention(cache, q.cuda(), ctx_t, TAU, num_splits=s, status=st).cpu().numpy()
        assert st.item() == 0
        ma, rl = gu.attention_errors(got, ref)
        print(f"kind={kind} bits={bits} g={hq // hkv} splits={s}: max-abs {ma:.3e} rel-L2 {rl:.3e}")
        assert ma <= MAX_ABS and rl <= REL_L2


@pytest.mark.parametrize("kind,bits,v_scale", [(0, 2, (300.0, 3000.0)), (1, 4, (1e-3, 4e3))])
def test_chunk_large_and_spread_value_scales(kind, bits, v_scale):
    """Value scales far above 1 and spread over many binades: the kernel carries
    e * scale in fp16, so it keeps the scales' running maximum exponent out of it."""
    n_q, bsz, hq, hkv, cap = 16, 2, 8, 2, 700
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=41 + bits, device="cpu", v_scale_range=v_scale)
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors={k: v.cuda() for k, v in c.items()})
    q = _chunk_queries(bsz, n_q, hq, seed=43).contiguous()
    ctx = [700, 333]
    cn = {name: t.numpy() for name, t in c.items()}
    cn["k_meta"] = cn["k_meta"].view(np.uint16)
    cn["v_meta"] = cn["v_meta"].view(np.uint16)
    ref = orc.chunk_attention(cn, q.numpy().astype(np.float64), ctx, TAU, kind, bits, hkv)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = dq.chunk_attention(cache, q.cuda(), torch.tensor(ctx, dtype=torch.int32, device="cuda"), TAU,
                             num_splits=1, status=st).cpu().numpy()
    assert st.item() == 0
    assert np.all(np.isfinite(got))
    scale = float(np.abs(ref).max())
    ma, rl = gu.attention_errors(got, ref)
    print(f"kind={kind} bits={bits} v_scale={v_scale}: max|ref| {scale:.3g} max-abs {ma:.3e} rel-L2 {rl:.3e}")
    # the bar scales with the values: 2e-3 of the largest output magnitude
    assert ma <= MAX_ABS * max(1.0, scale) and rl <= REL_L2


def test_chunk_last_query_and_splits():
    """The chunk's last query is the decode query at the same context; the split count
    changes results only at fp32 rounding level; contexts above the capacity are
    clamped with the overflow bit."""
    kind, bits, hq, hkv, n_q = 1, 2, 8, 2, 16
    bsz, cap = 3, 1100
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=15, device="cpu")
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors={k: v.cuda() for k, v in c.items()})
    q = _chunk_queries(bsz, n_q, hq, seed=21).cuda()
    ctx = torch.tensor([1100, 9, 513], dtype=torch.int32, device="cuda")
    outs = [dq.chunk_attention(cache, q, ctx, TAU, num_splits=s) for s in (0, 1, 3, 7)]
    for o in outs[1:]:
        assert torch.allclose(o, outs[0], rtol=0, atol=5e-5), (o - outs[0]).abs().max()
    # The last query through the decode call: the two kernels share no arithmetic (the
    # decode kernel rounds probabilities to 16-bit limbs, the chunk kernel carries them
    # as fp16 hi + lo), so each is held to the oracle at the bar.
    dec = dq.decode_attention(cache, q[:, n_q - 1].contiguous(), ctx, TAU)
    cn = {name: t.numpy() for name, t in c.items()}
    cn["k_meta"] = cn["k_meta"].view(np.uint16)
    cn["v_meta"] = cn["v_meta"].view(np.uint16)
    ref = orc.decode_attention(cn, q[:, n_q - 1].cpu().numpy().astype(np.float64), ctx.tolist(), TAU, kind, bits, hkv)
    for got in (outs[0][:, n_q - 1], dec):
        ma, rl = gu.attention_errors(got.cpu().numpy(), ref)
        assert ma <= MAX_ABS and rl <= REL_L2, (ma, rl)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    over = dq.chunk_attention(cache, q, torch.tensor([5000, 9, 513], dtype=torch.int32, device="cuda"), TAU,
                              status=st)
    torch.cuda.synchronize()
    assert st.item() & dq.STATUS_CTX_OVERFLOW
    assert torch.equal(over, outs[0])


def test_chunk_paged_equals_contiguous():
    kind, bits, hq, hkv, n_q, page = 0, 2, 16, 2, 16, 64
    bsz, cap = 2, 512
    pps = cap // page
    num_pages = bsz * pps + 3
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=19, device="cuda")
    flat = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=c)
    bt = torch.randperm(num_pages, generator=torch.Generator().manual_seed(2))[:bsz * pps].view(bsz, pps)
    bt = bt.to(torch.int32)
    pools = {}
    for name, t in c.items():
        pool = torch.zeros((num_pages, hkv, page) + tuple(t.shape[3:]), dtype=t.dtype, device="cuda")
        for b in range(bsz):
            for p in range(pps):
                pool[int(bt[b, p])] = t[b, :, p * page:(p + 1) * page]
        pools[name] = pool
    paged = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=pools, page_size=page, num_pages=num_pages,
                           block_table=bt)
    q = _chunk_queries(bsz, n_q, hq, seed=5).cuda()
    ctx = torch.tensor([512, 200], dtype=torch.int32, device="cuda")
    a = dq.chunk_attention(flat, q, ctx, TAU)
    b = dq.chunk_attention(paged, q, ctx, TAU)
    assert torch.equal(a, b)


@pytest.mark.parametrize("kind,bits,batch,hq,hkv,ctx", [
    (0, 2, 32, 64, 8, 8192),               # Qwen3-32B-shaped layer, QuEST 2-bit, 16-token chunk
    (0, 2, 16, 32, 8, 2048),               # Qwen3-8B shapes, last chunk of a 2048-token sequence
])
def test_chunk_full_size_sampled(kind, bits, batch, hq, hkv, ctx):
    """Full-size random caches; the oracle checks a sample of (sequence, KV head) pairs."""
    n_q = 16
    c = gen.random_cache(batch, hkv, ctx, kind, bits, seed=ctx + 3, device="cuda")
    cache = dq.PackedCache(batch, hkv, ctx, kind, bits, tensors=c)
    q = (torch.randn(batch, n_q, hq, 128, generator=torch.Generator(device="cuda").manual_seed(12),
                     device="cuda") * 2.0).contiguous()
    ctx_t = torch.full((batch,), ctx, dtype=torch.int32, device="cuda")
    ctx_t[-1] = ctx - 77                                       # ragged tail on one sequence
    out = dq.chunk_attention(cache, q, ctx_t, TAU).cpu().numpy()
    gsz = hq // hkv
    qn = q.cpu().numpy().astype(np.float64)
    ctx_h = ctx_t.cpu().numpy()
    for (b, kv) in [(0, 0), (batch - 1, hkv - 1), (batch // 2, 3 % hkv)]:
        one = {name: t[b:b + 1, kv:kv + 1].cpu().numpy() for name, t in c.items()}
        one["k_meta"] = one["k_meta"].view(np.uint16)
        one["v_meta"] = one["v_meta"].view(np.uint16)
        ref = orc.chunk_attention(one, qn[b:b + 1, :, kv * gsz:(kv + 1) * gsz], [int(ctx_h[b])], TAU, kind, bits, 1)
        ma, rl = gu.attention_errors(out[b:b + 1, :, kv * gsz:(kv + 1) * gsz], ref)
        assert ma <= MAX_ABS and rl <= REL_L2, (b, kv, ma, rl)


def test_chunk_after_gpu_append_end_to_end():
    """The pages' chunked forward on the tiny workload: the GPU appends the last 16
    tokens of a 256-token sequence after a 240-token history (both bf16, post-RoPE,
    through the key transform), maps the chunk's queries, and runs chunk attention;
    the oracle runs the same steps on the CPU.  Codes may differ by one step within
    1e-4 Delta of a boundary, which the attention bar absorbs."""
    w = TINY
    kind, bits, hq, hkv, n_q = 0, 2, 4, 1, 16
    tk, tinv = gen.transforms(w)
    k = gen.keys(w, 0, 1, 0, 256)
    v = gen.values(w, 0, 1, 0, 256)
    oc = orc.empty_cache(1, hkv, 256, kind, bits)
    assert orc.quantize_append(oc, gu.to_numpy64(k), gu.to_numpy64(v), [0], kind, bits, QUEST_ALPHA[bits],
                               tk=tk.astype(np.float64)) == 0
    cache = dq.PackedCache(1, hkv, 256, kind, bits, QUEST_ALPHA[bits])
    tk_d = torch.from_numpy(tk).cuda()
    dq.quantize_append(cache, k[:, :240].contiguous().cuda(), v[:, :240].contiguous().cuda(),
                       torch.tensor([0], dtype=torch.int32, device="cuda"), tk_d)
    dq.quantize_append(cache, k[:, 240:].contiguous().cuda(), v[:, 240:].contiguous().cuda(),
                       torch.tensor([240], dtype=torch.int32, device="cuda"), tk_d)
    q = torch.randn(1, n_q, hq, 128, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    qt = dq.transform_query(q.view(n_q, hq, 128).cuda(), torch.from_numpy(tinv).cuda(), hkv)
    got = dq.chunk_attention(cache, qt.view(1, n_q, hq, 128), torch.tensor([256], dtype=torch.int32,
                                                                           device="cuda"), TAU).cpu().numpy()
    qt_ref = orc.transform_query(gu.to_numpy64(q.view(n_q, hq, 128)), tinv.astype(np.float64), hkv)
    ref = orc.chunk_attention(oc, qt_ref.reshape(1, n_q, hq, 128), [256], TAU, kind, bits, hkv)
    ma, rl = gu.attention_errors(got, ref)
    assert ma <= MAX_ABS and rl <= REL_L2, (ma, rl)


def test_chunk_bad_page_entries():
    """A block-table entry outside the pool: chunk attention leaves those positions out
    (every query of the chunk) and raises the bad-page status bit."""
    kind, bits, hq, hkv, bsz, cap, page, n_q = 1, 2, 8, 2, 2, 512, 128, 16
    pps = cap // page
    num_pages = bsz * pps
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=7, device="cuda")
    bt = torch.randperm(num_pages, generator=torch.Generator().manual_seed(4))[:bsz * pps].view(bsz, pps)
    bt = bt.to(torch.int32)
    pools = {}
    for name, t in c.items():
        pool = torch.zeros((num_pages, hkv, page) + tuple(t.shape[3:]), dtype=t.dtype, device="cuda")
        for b in range(bsz):
            for p in range(pps):
                pool[int(bt[b, p])] = t[b, :, p * page:(p + 1) * page]
        pools[name] = pool
    bad = bt.clone()
    bad[1, 2] = num_pages                                   # positions 256..383 of sequence 1
    paged = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=pools, page_size=page, num_pages=num_pages,
                           block_table=bad)
    q = _chunk_queries(bsz, n_q, hq, seed=9)
    ctx = [512, 512]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = dq.chunk_attention(paged, q.cuda(), torch.tensor(ctx, dtype=torch.int32, device="cuda"), TAU,
                             status=st).cpu().numpy()
    torch.cuda.synchronize()
    assert st.item() & dq.STATUS_BAD_PAGE
    gsz = hq // hkv
    worst = 0.0
    for b in range(bsz):
        for kv in range(hkv):
            sel = {name: t[b, kv].cpu().numpy() for name, t in c.items()}
            for i in range(n_q):
                last = ctx[b] - n_q + i
                keep = np.arange(last + 1)
                if b == 1:
                    keep = keep[(keep < 256) | (keep >= 384)]
                ref = orc.decode_attention_pair(sel["k_codes"][keep], sel["k_meta"][keep].view(np.uint16),
                                                sel["v_codes"][keep], sel["v_meta"][keep].view(np.uint16),
                                                q[b, i, kv * gsz:(kv + 1) * gsz].numpy().astype(np.float64), TAU,
                                                kind, bits)
                ma, rl = gu.attention_errors(got[b, i, kv * gsz:(kv + 1) * gsz], ref)
                worst = max(worst, ma)
                assert ma <= MAX_ABS and rl <= REL_L2, (b, kv, i, ma, rl)
    print(f"bad page: worst max-abs {worst:.3e}")
