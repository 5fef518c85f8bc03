"""Helpers shared by the GPU parity tests: moving caches between the oracle's numpy
layout and the library's tensors, and the comparison rules the parity bar states."""
import numpy as np
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc


def to_numpy64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def cache_to_gpu(ocache, kind, bits, alpha=0.0, rank_lo=2, rank_hi=125) -> dq.PackedCache:
    b, h, t, _ = ocache["k_codes"].shape
    tens = {k: torch.from_numpy(np.ascontiguousarray(v.view(np.int16) if v.dtype == np.uint16 else v)).cuda()
            for k, v in ocache.items()}
    return dq.PackedCache(b, h, t, kind, bits, alpha, rank_lo, rank_hi, tensors=tens)


def cache_to_numpy(cache: dq.PackedCache):
    return {"k_codes": cache.k_codes.cpu().numpy(), "v_codes": cache.v_codes.cpu().numpy(),
            "k_meta": cache.k_meta.cpu().numpy().view(np.uint16),
            "v_meta": cache.v_meta.cpu().numpy().view(np.uint16)}


def fp16_midpoint_distance(pre):
    """|pre - nearest midpoint between two adjacent fp16 values| (float64)."""
    pre = np.asarray(pre, np.float64)
    r = orc.fp16_round(pre)
    h = np.abs(r).astype(np.float16)
    up = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h, np.float16(0)).astype(np.float64)
    a = np.abs(r)
    return np.minimum(np.abs(np.abs(pre) - (a + up) / 2), np.abs(np.abs(pre) - (a + dn) / 2))


def quest_boundary_distance(x, delta, bits):
    """Distance of each x to the nearest decision threshold j*Delta."""
    half = 1 << (bits - 1)
    d = np.asarray(delta, np.float64)[..., None]
    j = np.clip(np.round(x / np.where(d == 0, 1, d)), -(half - 1), half - 1)
    return np.abs(x - j * d)


def affine_boundary_distance(x, scale, zero, bits):
    levels = (1 << bits) - 1
    s = np.asarray(scale, np.float64)[..., None]
    z = np.asarray(zero, np.float64)[..., None]
    j = np.clip(np.floor((x - z) / np.where(s == 0, 1, s)), 0, levels - 1)
    return np.abs(x - (z + (j + 0.5) * s))


def attention_errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    max_abs = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel_l2


def check_key_rows(oc, gc, x, kind, bits, start, alpha):
    """End-to-end rule for the key side of an append: oracle cache oc and GPU cache gc
    (numpy dicts), x = the oracle's transformed keys [B, n, Hkv, 128] written at
    start[b] + t.  Meta may differ by one fp16 ulp only where the oracle's pre-rounding
    value lies within 1e-4 * Delta of an fp16 midpoint; codes (against the oracle's
    quantizer given the GPU's meta) by +-1 only within 1e-4 * Delta of a threshold.
    Returns (meta flips, code differences, values near a boundary)."""
    bsz, n = x.shape[:2]
    meta_flips = code_diffs = near = 0
    for b in range(bsz):
        sl = slice(start[b], start[b] + n)
        om = oc["k_meta"][b, :, sl].transpose(1, 0, 2)
        gm = gc["k_meta"][b, :, sl].transpose(1, 0, 2)
        xo = x[b]
        flip = np.any(om != gm, axis=-1)
        if flip.any():
            if kind == orc.QUEST_INT:
                dist = fp16_midpoint_distance(orc.quest_step_prerounding(xo, bits, alpha))
                assert np.all(dist[flip] <= 1e-4 * orc.fp16_value(om[..., 0])[flip])
            else:
                sp, lo = orc.affine_prerounding(xo, bits, 2, 125)
                dd = np.minimum(fp16_midpoint_distance(sp), fp16_midpoint_distance(lo))
                assert np.all(dd[flip] <= 1e-4 * orc.fp16_value(om[..., 0])[flip])
            meta_flips += int(flip.sum())
        gmv = orc.fp16_value(gm)
        if kind == orc.QUEST_INT:
            ref = orc.quest_codes(xo, gmv[..., 0], bits)
            dist = quest_boundary_distance(xo, gmv[..., 0], bits)
        else:
            ref = orc.affine_codes(xo, gmv[..., 0], gmv[..., 1], bits)
            dist = affine_boundary_distance(xo, gmv[..., 0], gmv[..., 1], bits)
        step = np.broadcast_to(gmv[..., 0][..., None], dist.shape)
        got = orc.unpack_codes(gc["k_codes"][b, :, sl].transpose(1, 0, 2), bits)
        diff = got.astype(np.int32) - ref.astype(np.int32)
        assert np.all(np.abs(diff) <= 1)
        off = diff != 0
        assert np.all(dist[off] <= 1e-4 * step[off]), "code differs away from a boundary"
        code_diffs += int(off.sum())
        near += int((dist <= 1e-4 * step).sum())
    return meta_flips, code_diffs, near


def append_history(cache, w, n_tokens, tk, layer=0, chunk=4096):
    """Fill positions 0 .. n_tokens-1 of every sequence with the GPU's own appends of the
    workload's synthetic keys and values (chunks of `chunk` tokens; tk a device tensor)."""
    t = 0
    status = torch.zeros(1, dtype=torch.int32, device=cache.device)
    while t < n_tokens:
        n = min(chunk, n_tokens - t)
        k = gen_keys(w, t, n, layer, cache.device)
        v = gen_values(w, t, n, layer, cache.device)
        sp = torch.full((w.batch,), t, dtype=torch.int32, device=cache.device)
        dq.quantize_append(cache, k, v, sp, tk, status)
        t += n
    torch.cuda.synchronize()
    return int(status.item())


def gen_keys(w, t0, n, layer, device):
    from synth import gen
    return gen.keys(w, 0, w.batch, t0, n, layer=layer, device=device)


def gen_values(w, t0, n, layer, device):
    from synth import gen
    return gen.values(w, 0, w.batch, t0, n, layer=layer, device=device)


def decode_vs_oracle(cache_np, q_t, ctx, tau, kind, bits, num_kv_heads, out, pairs=None):
    """Oracle decode (fp64) of the (sequence, KV head) pairs listed (all when None) over the
    given numpy cache, against the GPU output `out` [B, Hq, 128]; returns the worst
    (max-abs, rel-L2) over the pairs and the number of pairs checked."""
    import oracle.wushkv_oracle as orc_
    bsz, hq, _ = q_t.shape
    g = hq // num_kv_heads
    if pairs is None:
        pairs = [(b, kv) for b in range(bsz) for kv in range(num_kv_heads)]
    worst_ma = worst_rl = 0.0
    for (b, kv) in pairs:
        n = int(min(ctx[b], cache_np["k_codes"].shape[2]))
        ref = orc_.decode_attention_pair(cache_np["k_codes"][b, kv, :n], cache_np["k_meta"][b, kv, :n],
                                         cache_np["v_codes"][b, kv, :n], cache_np["v_meta"][b, kv, :n],
                                         q_t[b, kv * g:(kv + 1) * g], tau, kind, bits)
        ma, rl = attention_errors(out[b, kv * g:(kv + 1) * g], ref)
        worst_ma, worst_rl = max(worst_ma, ma), max(worst_rl, rl)
    return worst_ma, worst_rl, len(pairs)
