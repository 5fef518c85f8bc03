"""Quantize-append at full workload sizes, in the launch configuration the benchmark
times, checked on a deterministic sample of (sequence, token, KV head) groups that the
oracle computes one by one: value codes and meta bit-exact; key meta flips only within
1e-4 * Delta of an fp16 rounding midpoint; key codes off by one only within 1e-4 * Delta
of a decision threshold (counts printed).
"""
import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QUEST_ALPHA, QWEN8B_DECODE, QWEN8B_SWEEP, QWEN32B_STACK
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _check_sample(w, cache, k, v, tk, start, samples):
    qs = w.quant
    alpha = qs.clip_alpha if qs.kind == orc.QUEST_INT else 0.0
    got = {name: t.cpu() for name, t in cache.tensors().items()}
    flips = diffs = 0
    for (b, t, h) in samples:
        pos = start[b] + t
        kx = orc.transform_keys(gu.to_numpy64(k[b, t, h][None, None, :]),
                                tk[h:h + 1].astype(np.float64))[0, 0]
        vx = gu.to_numpy64(v[b, t, h])
        for side, x in (("k", kx), ("v", vx)):
            codes = orc.quantize_groups(x[None], qs.kind, qs.bits, alpha, qs.rank_lo, qs.rank_hi)
            ref_codes, ref_meta = codes
            gm = got[f"{side}_meta"][b, h, pos].numpy().view(np.uint16)
            gc = got[f"{side}_codes"][b, h, pos].numpy()
            if side == "v":
                assert np.array_equal(gm, ref_meta[0]), (b, t, h)
                assert np.array_equal(gc, orc.pack_codes(ref_codes, qs.bits)[0]), (b, t, h)
                continue
            gmv = orc.fp16_value(gm)
            if not np.array_equal(gm, ref_meta[0]):
                if qs.kind == orc.QUEST_INT:
                    d = gu.fp16_midpoint_distance(orc.quest_step_prerounding(x, qs.bits, alpha))
                else:
                    sp, lo = orc.affine_prerounding(x, qs.bits, qs.rank_lo, qs.rank_hi)
                    d = min(gu.fp16_midpoint_distance(sp), gu.fp16_midpoint_distance(lo))
                assert d <= 1e-4 * gmv[0], (b, t, h, "meta")
                flips += 1
            if qs.kind == orc.QUEST_INT:
                ref = orc.quest_codes(x, gmv[0], qs.bits)
                dist = gu.quest_boundary_distance(x, gmv[0], qs.bits)
            else:
                ref = orc.affine_codes(x, gmv[0], gmv[1], qs.bits)
                dist = gu.affine_boundary_distance(x, gmv[0], gmv[1], qs.bits)
            out = orc.unpack_codes(gc[None], qs.bits)[0].astype(np.int32)
            diff = out - ref.astype(np.int32)
            assert np.all(np.abs(diff) <= 1) and np.all(dist[diff != 0] <= 1e-4 * gmv[0]), (b, t, h, "codes")
            diffs += int((diff != 0).sum())
    return flips, diffs


def _samples(w, n, count, seed):
    rng = np.random.default_rng(seed)
    s = [(0, 0, 0), (w.batch - 1, n - 1, w.num_kv_heads - 1)]
    s += [(int(rng.integers(w.batch)), int(rng.integers(n)), int(rng.integers(w.num_kv_heads)))
          for _ in range(count)]
    return s


@pytest.mark.parametrize("w", [QWEN8B_SWEEP(2), QWEN8B_SWEEP(3), QWEN8B_SWEEP(4)], ids=lambda w: w.name)
def test_chunk_append_full_size_sampled(w):
    """The 2048-token chunk x 16 sequences x 8 KV heads of the bit-width sweep, appended at
    position 30720 of a 32768-token cache (the tensor-core path)."""
    qs = w.quant
    n = w.append_tokens
    tk = gen.transforms(w)[0]
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha)
    k = gen.keys(w, 0, w.batch, w.history, n, device="cuda")
    v = gen.values(w, 0, w.batch, w.history, n, device="cuda")
    start = [w.history] * w.batch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append(cache, k, v, torch.tensor(start, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(tk).cuda(), st)
    torch.cuda.synchronize()
    assert st.item() == 0
    flips, diffs = _check_sample(w, cache, k.cpu(), v.cpu(), tk, start, _samples(w, n, 48, 1))
    print(f"{w.name}: key meta flips {flips}, key code diffs {diffs} in 50 sampled groups")


@pytest.mark.parametrize("w,layer", [(QWEN32B_STACK, 0), (QWEN32B_STACK, 63), (QWEN8B_DECODE, 0)],
                         ids=["qwen32b_layer0", "qwen32b_layer63", "qwen8b_decode_token"])
def test_step_append_full_size_sampled(w, layer):
    """One decode step's append: the Qwen3-32B-shaped layer's 16-token chunk (512 rows,
    tensor-core path) at position 8176, and the Qwen3-8B-shaped layer's single token per
    sequence (16 rows, one-warp-per-group path) at position 32767."""
    qs = w.quant
    n = w.append_tokens
    tk = gen.transforms(w, layer)[0]
    cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha, qs.rank_lo, qs.rank_hi)
    k = gen.keys(w, 0, w.batch, w.history, n, layer=layer, device="cuda")
    v = gen.values(w, 0, w.batch, w.history, n, layer=layer, device="cuda")
    start = [w.history] * w.batch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append(cache, k, v, torch.tensor(start, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(tk).cuda(), st)
    torch.cuda.synchronize()
    assert st.item() == 0
    flips, diffs = _check_sample(w, cache, k.cpu(), v.cpu(), tk, start, _samples(w, n, 48, 2 + layer))
    print(f"{w.name} layer {layer}: key meta flips {flips}, key code diffs {diffs} in 50 sampled groups")
