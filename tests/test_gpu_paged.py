"""Paged cache layout (pools of pages + block table): every kernel must give exactly
what it gives on the contiguous layout holding the same rows, and decode over a paged
cache must match the oracle on the gathered cache.  Entries outside the pool are
skipped with the bad-page status bit."""
import math

import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QUEST_ALPHA, QWEN8B_DECODE
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
TAU = 1.0 / math.sqrt(128)


def _block_table(batch, pps, num_pages, seed):
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed))[:batch * pps]
    return perm.view(batch, pps).to(torch.int32)


def _paged_from(c, block_table, page_size, num_pages):
    """Scatter a contiguous cache dict into page pools (test-side layout change only)."""
    out = {}
    for name, t in c.items():
        pool = torch.zeros((num_pages, t.shape[1], page_size) + tuple(t.shape[3:]), dtype=t.dtype, device=t.device)
        for b in range(block_table.shape[0]):
            for p in range(block_table.shape[1]):
                pool[int(block_table[b, p])] = t[b, :, p * page_size:(p + 1) * page_size]
        out[name] = pool
    return out


def _gather(cache):
    bt = cache.block_table.cpu().numpy()
    return {name: torch.from_numpy(orc.gather_paged(t.cpu().numpy(), bt, cache.page_size))
            for name, t in cache.tensors().items()}


@pytest.mark.parametrize("page_size", [16, 64, 256, 512])
@pytest.mark.parametrize("kind,bits,hq,hkv", [(1, 2, 8, 2), (0, 4, 16, 2), (0, 3, 8, 2)])
def test_paged_decode_equals_contiguous(page_size, kind, bits, hq, hkv):
    bsz, cap = 3, 1024
    pps = cap // page_size
    num_pages = bsz * pps + 5
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=page_size + bits, device="cuda")
    flat = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=c)
    bt = _block_table(bsz, pps, num_pages, seed=page_size)
    paged = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=_paged_from(c, bt, page_size, num_pages),
                           page_size=page_size, num_pages=num_pages, block_table=bt)
    q = torch.randn(bsz, hq, 128, generator=torch.Generator().manual_seed(9)).cuda() * 2.0
    ctx = torch.tensor([1024, 300, 777], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for ns in (0, 2):
        a = dq.decode_attention(flat, q, ctx, TAU, num_splits=ns)
        b = dq.decode_attention(paged, q, ctx, TAU, num_splits=ns, status=st)
        torch.cuda.synchronize()
        assert torch.equal(a, b), (ns, (a - b).abs().max().item())
    assert st.item() == 0
    # the oracle on the gathered cache
    g = _gather(paged)
    out = b.cpu().numpy()
    gsz = hq // hkv
    for s in range(bsz):
        for kv in range(hkv):
            n = int(ctx[s])
            ref = orc.decode_attention_pair(g["k_codes"][s, kv, :n].numpy(), g["k_meta"][s, kv, :n].numpy().view(np.uint16),
                                            g["v_codes"][s, kv, :n].numpy(), g["v_meta"][s, kv, :n].numpy().view(np.uint16),
                                            q[s, kv * gsz:(kv + 1) * gsz].cpu().numpy().astype(np.float64), TAU, kind, bits)
            ma, rl = gu.attention_errors(out[s, kv * gsz:(kv + 1) * gsz], ref)
            assert ma <= 2e-3 and rl <= 1e-2, (s, kv, ma, rl)


@pytest.mark.parametrize("page_size", [16, 128, 256])
@pytest.mark.parametrize("bsz,n,dtype", [(2, 300, torch.bfloat16), (16, 1, torch.bfloat16), (2, 40, torch.float32)],
                         ids=["bulk", "step", "fp32"])
def test_paged_append_equals_contiguous(page_size, bsz, n, dtype):
    """Tensor-core (> 64 bf16 rows), one-warp-per-group (<= 64 rows) and fp32 appends."""
    w = QWEN8B_DECODE
    hkv, cap = 2, 512
    pps = cap // page_size
    num_pages = bsz * pps + 3
    start = [(37 * b) % 150 for b in range(bsz)]
    tk = torch.from_numpy(gen.transforms(w)[0][:hkv].copy()).cuda()
    k = gen.keys(w, 0, bsz, start, n)[:, :, :hkv].contiguous().to(dtype).cuda()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous().to(dtype).cuda()
    sp = torch.tensor(start, dtype=torch.int32, device="cuda")
    for kind, bits in ((0, 2), (1, 3)):
        alpha = QUEST_ALPHA[bits] if kind == 0 else 0.0
        flat = dq.PackedCache(bsz, hkv, cap, kind, bits, alpha)
        bt = _block_table(bsz, pps, num_pages, seed=bits)
        paged = dq.PackedCache(bsz, hkv, cap, kind, bits, alpha, page_size=page_size, num_pages=num_pages,
                               block_table=bt)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        dq.quantize_append(flat, k, v, sp, tk)
        dq.quantize_append(paged, k, v, sp, tk, st)
        torch.cuda.synchronize()
        assert st.item() == 0
        g = _gather(paged)
        for name, t in flat.tensors().items():
            assert torch.equal(t.cpu(), g[name]), (kind, bits, name)


def test_bad_page_entries():
    """A block-table entry outside the pool: the append skips those rows and decode
    leaves them out, both with the bad-page status bit."""
    kind, bits, hq, hkv, bsz, cap, page = 1, 2, 8, 2, 2, 512, 128
    pps = cap // page
    num_pages = bsz * pps
    c = gen.random_cache(bsz, hkv, cap, kind, bits, seed=3, device="cuda")
    bt = _block_table(bsz, pps, num_pages, seed=1)
    pools = _paged_from(c, bt, page, num_pages)
    bad = bt.clone()
    bad[1, 2] = num_pages                                   # positions 256..383 of sequence 1
    paged = dq.PackedCache(bsz, hkv, cap, kind, bits, tensors=pools, page_size=page, num_pages=num_pages,
                           block_table=bad)
    q = torch.randn(bsz, hq, 128, generator=torch.Generator().manual_seed(2)).cuda()
    ctx = torch.tensor([512, 512], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = dq.decode_attention(paged, q, ctx, TAU, status=st).cpu().numpy()
    torch.cuda.synchronize()
    assert st.item() & dq.STATUS_BAD_PAGE
    keep = np.r_[0:256, 384:512]                            # sequence 1 without the bad page
    gsz = hq // hkv
    for kv in range(hkv):
        sel = {name: t[1, kv].cpu().numpy()[keep] for name, t in c.items()}
        ref = orc.decode_attention_pair(sel["k_codes"], sel["k_meta"].view(np.uint16), sel["v_codes"],
                                        sel["v_meta"].view(np.uint16),
                                        q[1, kv * gsz:(kv + 1) * gsz].cpu().numpy().astype(np.float64), TAU, kind, bits)
        ma, rl = gu.attention_errors(out[1, kv * gsz:(kv + 1) * gsz], ref)
        assert ma <= 2e-3 and rl <= 1e-2, (kv, ma, rl)
    # append into the bad page: nothing written, status raised
    w = QWEN8B_DECODE
    k = gen.keys(w, 0, bsz, [300, 300], 1)[:, :, :hkv].contiguous().cuda()
    v = gen.values(w, 0, bsz, [300, 300], 1)[:, :, :hkv].contiguous().cuda()
    before = {name: t.clone() for name, t in paged.tensors().items()}
    st.zero_()
    dq.quantize_append(paged, k, v, torch.tensor([300, 300], dtype=torch.int32, device="cuda"), None, st)
    torch.cuda.synchronize()
    assert st.item() & dq.STATUS_BAD_PAGE
    page0 = int(bt[0, 2])                                   # sequence 0 still wrote its row
    assert not torch.equal(before["k_codes"][page0], paged.k_codes[page0])
