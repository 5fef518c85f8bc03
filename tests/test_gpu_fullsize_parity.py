"""Full-size parity on the workloads' own synthetic data, with nothing sampled.

* Quantize-append of the bit-width sweep's 2048-token chunk (16 sequences x 8 KV heads,
  QuEST 2/3/4-bit, the tensor-core path in the benchmark's launch configuration): every
  one of the 262,144 groups against the oracle's append of the same bf16 keys and T_k.
  Value codes and meta bit-exact; key meta flips only within 1e-4 * Delta of an fp16
  rounding midpoint and key codes off by one only within 1e-4 * Delta of a threshold
  (both counts asserted and printed).
* Decode attention over caches the GPU's own appends built from the workloads' keys
  (outlier channels, RoPE) and values (heavy channels): the Qwen3-8B-shaped layer at
  context 32768 and the long-context layer at 131072, every (sequence, KV head) pair
  against the oracle on the same codes, max-abs <= 2e-3 and relative L2 <= 1e-2.
* The tensor-core key epilogue alone, bit-exact: bf16 keys placed exactly on QuEST
  thresholds and on affine half-way points go through the tensor-core append with an
  explicit identity T_k and with a (signed) permutation T_k, both exact in the first
  bf16 plane, so the quantizer sees exactly the oracle's x.
"""
import math

import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QUEST_ALPHA, QWEN8B_DECODE, QWEN8B_LONG, QWEN8B_SWEEP
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
TAU = 1.0 / math.sqrt(128)
MAX_ABS, REL_L2 = 2e-3, 1e-2


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_chunk_append_every_group(bits):
    w = QWEN8B_SWEEP(bits)
    qs = w.quant
    n = w.append_tokens
    tk = gen.transforms(w)[0]
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha)
    k = gen.keys(w, 0, w.batch, w.history, n, device="cuda")
    v = gen.values(w, 0, w.batch, w.history, n, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append(cache, k, v, torch.full((w.batch,), w.history, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(tk).cuda(), st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rows = slice(w.history, w.history + n)
    gc = {name: t[:, :, rows].cpu().numpy() for name, t in cache.tensors().items()}
    for name in ("k_meta", "v_meta"):
        gc[name] = gc[name].view(np.uint16)
    k64, v64 = gu.to_numpy64(k), gu.to_numpy64(v)
    del k, v
    oc = orc.empty_cache(w.batch, w.num_kv_heads, n, qs.kind, qs.bits)
    assert orc.quantize_append(oc, k64, v64, [0] * w.batch, qs.kind, qs.bits, qs.clip_alpha,
                               tk=tk.astype(np.float64)) == 0
    for name in ("v_codes", "v_meta"):
        bad = int((oc[name] != gc[name]).sum())
        assert bad == 0, f"{name}: {bad} bytes differ"
    x = orc.transform_keys(k64, tk.astype(np.float64))
    del k64, v64
    flips, diffs, near = gu.check_key_rows(oc, gc, x, qs.kind, qs.bits, [0] * w.batch, qs.clip_alpha)
    groups = w.batch * n * w.num_kv_heads
    print(f"{w.name}: {groups} groups; key meta flips {flips}, key code diffs {diffs}, "
          f"values within 1e-4 Delta of a threshold {near}")


@pytest.mark.parametrize("w", [QWEN8B_DECODE, QWEN8B_LONG], ids=lambda w: w.name)
def test_decode_every_pair_on_appended_cache(w):
    qs = w.quant
    tk, tinv = gen.transforms(w)
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, qs.rank_lo, qs.rank_hi)
    assert gu.append_history(cache, w, w.ctx, torch.from_numpy(tk).cuda()) == 0
    q = gen.queries(w, device="cuda").contiguous()
    q_t = dq.transform_query(q, torch.from_numpy(tinv).cuda(), w.num_kv_heads)
    ctx = torch.full((w.batch,), w.ctx, dtype=torch.int32, device="cuda")
    ctx[-1] = w.ctx - 77                                     # a ragged tail on one sequence
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = dq.decode_attention(cache, q_t, ctx, TAU, status=st).cpu().numpy()
    assert st.item() == 0
    cn = gu.cache_to_numpy(cache)
    del cache
    ma, rl, npairs = gu.decode_vs_oracle(cn, q_t.cpu().numpy().astype(np.float64), ctx.cpu().numpy(), TAU,
                                         qs.kind, qs.bits, w.num_kv_heads, out)
    print(f"{w.name}: {npairs} pairs, worst max-abs {ma:.3e}, worst rel-L2 {rl:.3e}")
    assert npairs == w.batch * w.num_kv_heads
    assert ma <= MAX_ABS and rl <= REL_L2


def _affine_groups_on_halfway_points(n_groups, bits, seed):
    """bf16 groups whose percentile-affine grid has bf16 half-way points, with elements
    placed exactly on them: ranks 2 and 125 are set to -R and R with 2R = (2^b - 1) 2^-e,
    so scale = 2^-e and every threshold zero + (j + 1/2) scale is a short binary fraction;
    the other values lie strictly inside (-R, R) and a few of them are moved onto the
    thresholds (ties included, which round half to even)."""
    rng = np.random.default_rng(seed)
    levels = (1 << bits) - 1
    out = []
    for i in range(n_groups):
        e = int(rng.integers(-3, 3))
        r = levels * 2.0 ** (-e) / 2
        inner = rng.uniform(-r, r, 122)
        g = np.concatenate([[-r * 1.5, -r * 1.25, -r], inner, [r, r * 1.25, r * 1.5]])
        g = torch.from_numpy(g.astype(np.float32)).bfloat16().float().numpy()
        thr = [-r + (j + 0.5) * 2.0 ** (-e) for j in range(levels)]
        pos = rng.choice(np.arange(3, 125), size=len(thr), replace=False)
        g[pos] = np.asarray(thr, np.float32)
        out.append(rng.permutation(g))
    return np.stack(out).astype(np.float32)


def _perm_transform(seed, signs):
    rng = np.random.default_rng(seed)
    p = rng.permutation(128)
    t = np.zeros((128, 128), np.float32)
    t[np.arange(128), p] = rng.choice([-1.0, 1.0], 128) if signs else 1.0
    return t


@pytest.mark.parametrize("kind,bits", [(0, 2), (0, 3), (0, 4), (1, 2), (1, 3), (1, 4)])
def test_tc_key_epilogue_bitexact_on_thresholds(kind, bits):
    """Keys through the tensor-core append (256 rows of two KV heads, so more than the
    64 rows of the decode-step path) with T_k = I on head 0 and a permutation on head 1
    (signed for QuEST, whose thresholds are symmetric): x = T_k k is exact, so codes and
    meta must equal the oracle's bit for bit, on values that sit on decision thresholds."""
    n, hkv = 256, 2
    if kind == orc.QUEST_INT:
        from tests.test_gpu_append import _bf16_groups_on_thresholds
        groups = _bf16_groups_on_thresholds(n * hkv, bits, seed=300 + bits)
    else:
        groups = _affine_groups_on_halfway_points(n * hkv, bits, seed=400 + bits)
    # head 1 holds P^T applied to its groups, so that P k puts them back on the thresholds
    t1 = _perm_transform(500 + bits, signs=(kind == orc.QUEST_INT))
    k = groups.reshape(1, n, hkv, 128).copy()
    k[0, :, 1] = k[0, :, 1] @ t1                  # P^T g (P orthogonal, entries 0/+-1: exact)
    tk = np.stack([np.eye(128, dtype=np.float32), t1])
    vals = gen.fp32_groups((1, n, hkv, 128), seed=600 + bits, heavy_tail=False).numpy()
    kt = torch.from_numpy(k).bfloat16()
    vt = torch.from_numpy(vals).bfloat16()
    assert torch.equal(kt.float(), torch.from_numpy(k))          # the crafted keys are bf16 values
    alpha = QUEST_ALPHA[bits] if kind == orc.QUEST_INT else 0.0
    oc = orc.empty_cache(1, hkv, n, kind, bits)
    assert orc.quantize_append(oc, gu.to_numpy64(kt), gu.to_numpy64(vt), [0], kind, bits, alpha,
                               tk=tk.astype(np.float64)) == 0
    x = orc.transform_keys(gu.to_numpy64(kt), tk.astype(np.float64))
    assert np.array_equal(x.reshape(-1, 128), groups.astype(np.float64))   # back on the thresholds
    if kind == orc.QUEST_INT:
        d = orc.quest_meta(x, bits, alpha)
        half = 1 << (bits - 1)
        on = sum(int(np.isclose(x, j * d[..., None], rtol=0, atol=0).sum()) for j in range(-(half - 1), half))
    else:
        s, z = orc.affine_meta(x, bits, 2, 125)
        on = sum(int((x == z[..., None] + (j + 0.5) * s[..., None]).sum()) for j in range((1 << bits) - 1))
    assert on >= n * hkv                                          # the case really sits on thresholds
    cache = dq.PackedCache(1, hkv, n, kind, bits, alpha, 2, 125)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append(cache, kt.cuda(), vt.cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(tk).cuda(), st)
    torch.cuda.synchronize()
    assert st.item() == 0
    gc = gu.cache_to_numpy(cache)
    for name in ("k_meta", "k_codes", "v_meta", "v_codes"):
        bad = np.argwhere(oc[name] != gc[name])
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:3].tolist()}"
    print(f"kind={kind} bits={bits}: {on} key values on thresholds, all codes and meta bit-exact")
