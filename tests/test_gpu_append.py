"""GPU parity of wushkv_quantize_append against the CPU oracle.

* Quantizer alone (fp32 inputs, no transform): codes and fp16 meta bit-exact,
  including groups built to sit on decision thresholds and on fp16 rounding
  midpoints of the step/scale, which exercise the exact fallbacks.
* End to end (bf16 post-RoPE keys with outlier channels, random invertible T_k):
  value codes/meta bit-exact; key meta may differ by one fp16 ulp only where the
  oracle's pre-rounding value lies within 1e-4 * Delta of a rounding midpoint; key
  codes may differ by +-1 only where the oracle's x lies within 1e-4 * Delta of a
  decision threshold.  The counts are printed.
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


def _nearest_midpoint(pre):
    r = float(orc.fp16_round(pre))
    h = np.float16(abs(r))
    cands = [np.nextafter(h, np.float16(np.inf)), np.nextafter(h, np.float16(0))]
    mids = [(abs(r) + float(c)) / 2 for c in cands]
    return min(mids, key=lambda m: abs(m - abs(pre))) * np.sign(pre)


def craft_groups(x, kind, bits):
    """Make some groups hit thresholds / rounding midpoints exactly or nearly (oracle-side)."""
    x = x.copy()
    half = 1 << (bits - 1)
    levels = (1 << bits) - 1
    alpha = _alpha(kind, bits)
    g = x.reshape(-1, 128)
    for r in range(0, 24):                      # values exactly on thresholds
        xg = g[r].astype(np.float32)
        for _ in range(4):
            if kind == orc.QUEST_INT:
                d = float(orc.quest_meta(xg.astype(np.float64), bits, alpha))
                vals = [np.float32(j * d) for j in range(-(half - 1), half)]
            else:
                s, z = orc.affine_meta(xg.astype(np.float64), bits, 2, 125)
                vals = [np.float32(float(z) + (j + 0.5) * float(s)) for j in range(levels)]
            order = np.argsort(xg)
            mid_pos = order[10:10 + len(vals)]   # not among the extremes
            for p, v in zip(mid_pos, vals):
                xg[p] = v
        g[r] = xg
    for r in range(24, 48):                     # step / scale / zero next to an fp16 midpoint
        xg = g[r].astype(np.float64)
        if kind == orc.QUEST_INT:
            pre = float(orc.quest_step_prerounding(xg, bits, alpha))
        else:
            pre = float(orc.affine_prerounding(xg, bits, 2, 125)[0 if r % 2 else 1])
        if pre != 0:
            g[r] = (xg * (_nearest_midpoint(pre) / pre)).astype(np.float32)
    g[48] = 0.0                                  # Delta == 0 / scale == 0
    g[49] = 1.5
    return g.reshape(x.shape)


def _run_both(k, v, kind, bits, start, cap, tk=None):
    bsz, n, hkv, _ = k.shape
    alpha = _alpha(kind, bits)
    oc = orc.empty_cache(bsz, hkv, cap, kind, bits)
    o_status = orc.quantize_append(oc, gu.to_numpy64(k), gu.to_numpy64(v), start, kind, bits, alpha, 2, 125,
                                   tk=None if tk is None else tk.numpy().astype(np.float64))
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, alpha, 2, 125)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq.quantize_append(cache, k.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32, device="cuda"),
                       None if tk is None else tk.cuda(), status)
    torch.cuda.synchronize()
    return oc, o_status, gu.cache_to_numpy(cache), int(status.item())


@pytest.mark.parametrize("kind,bits", CASES)
def test_quantizer_bitexact_on_fp32_inputs(kind, bits):
    bsz, n, hkv, cap = 2, 300, 2, 333
    x = gen.fp32_groups((bsz, n, hkv, 128), seed=100 + 10 * kind + bits).numpy()
    v = gen.fp32_groups((bsz, n, hkv, 128), seed=200 + 10 * kind + bits, heavy_tail=False).numpy()
    x = craft_groups(x, kind, bits)
    oc, ost, gc, gst = _run_both(torch.from_numpy(x), torch.from_numpy(v), kind, bits, [0, 33], cap)
    assert ost == 0 and gst == 0
    for name in ("k_meta", "v_meta", "k_codes", "v_codes"):
        bad = np.argwhere(oc[name] != gc[name])
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:3].tolist()}"


def test_quantizer_status_bits():
    bsz, n, hkv, cap = 1, 8, 1, 6
    x = gen.fp32_groups((bsz, n, hkv, 128), seed=7).numpy()
    x[0, 1, 0, 5] = np.nan
    x[0, 2, 0, :] = 3.0e6                     # Delta overflows fp16
    oc, ost, gc, gst = _run_both(torch.from_numpy(x), torch.from_numpy(x.copy()), 0, 2, [0], cap)
    assert ost & orc.STATUS_CAPACITY and gst & dq.STATUS_CAPACITY          # rows 6, 7 do not fit
    assert gst & dq.STATUS_NONFINITE and gst & dq.STATUS_META_OVERFLOW
    good = [0, 3, 4, 5]
    for name in ("k_codes", "k_meta"):
        np.testing.assert_array_equal(oc[name][0, 0, good], gc[name][0, 0, good])


def _e2e_check(k, v, tk, kind, bits, start, cap):
    oc, ost, gc, gst = _run_both(k, v, kind, bits, start, cap, tk=tk)
    assert ost == 0 and gst == 0
    np.testing.assert_array_equal(oc["v_meta"], gc["v_meta"])
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    # key side, position by position
    alpha = _alpha(kind, bits)
    x = orc.transform_keys(gu.to_numpy64(k), tk.numpy().astype(np.float64))   # [B, n, H, 128]
    bsz, n, hkv, _ = k.shape
    meta_flips = code_diffs = near = 0
    for b in range(bsz):
        sl = slice(start[b], start[b] + n)
        om = oc["k_meta"][b, :, sl].transpose(1, 0, 2)       # [n, H, m]
        gm = gc["k_meta"][b, :, sl].transpose(1, 0, 2)
        xo = x[b]                                            # [n, H, 128]
        flip = np.any(om != gm, axis=-1)
        if flip.any():
            if kind == orc.QUEST_INT:
                pre = orc.quest_step_prerounding(xo, bits, alpha)
                dist = gu.fp16_midpoint_distance(pre)
                assert np.all(dist[flip] <= 1e-4 * orc.fp16_value(om[..., 0])[flip])
            else:
                sp, lo = orc.affine_prerounding(xo, bits, 2, 125)
                ds, dz = gu.fp16_midpoint_distance(sp), gu.fp16_midpoint_distance(lo)
                tol = 1e-4 * orc.fp16_value(om[..., 0])
                assert np.all(np.minimum(ds, dz)[flip] <= tol[flip])
            meta_flips += int(flip.sum())
        # reference codes: oracle x quantized with the meta the GPU stored
        gmv = orc.fp16_value(gm)
        if kind == orc.QUEST_INT:
            ref = orc.quest_codes(xo, gmv[..., 0], bits)
            dist = gu.quest_boundary_distance(xo, gmv[..., 0], bits)
            step = gmv[..., 0][..., None]
        else:
            ref = orc.affine_codes(xo, gmv[..., 0], gmv[..., 1], bits)
            dist = gu.affine_boundary_distance(xo, gmv[..., 0], gmv[..., 1], bits)
            step = gmv[..., 0][..., None]
        got = orc.unpack_codes(gc["k_codes"][b, :, sl].transpose(1, 0, 2), bits)
        diff = got.astype(np.int32) - ref.astype(np.int32)
        assert np.all(np.abs(diff) <= 1)
        off = diff != 0
        assert np.all(dist[off] <= 1e-4 * np.broadcast_to(step, dist.shape)[off]), "code differs away from a boundary"
        code_diffs += int(off.sum())
        near += int((dist <= 1e-4 * step).sum())
    print(f"kind={kind} bits={bits}: key meta flips {meta_flips}, key code diffs {code_diffs} "
          f"(values within 1e-4*Delta of a boundary: {near})")


@pytest.mark.parametrize("kind,bits", CASES)
def test_append_end_to_end_with_transform(kind, bits):
    w = QWEN8B_DECODE
    bsz, n, hkv, cap = 2, 200, 2, 260
    start = [0, 51]
    tk = torch.from_numpy(gen.transforms(w)[0][:hkv].copy())
    k = gen.keys(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    _e2e_check(k, v, tk, kind, bits, start, cap)


def test_append_identity_transform_equals_no_transform():
    """T_k = I reduces to plain quantization of the keys: both calls give the same cache."""
    w = QWEN8B_DECODE
    k = gen.keys(w, 0, 2, 0, 130)[:, :, :2].contiguous().cuda()
    v = gen.values(w, 0, 2, 0, 130)[:, :, :2].contiguous().cuda()
    eye = torch.eye(128).expand(2, 128, 128).contiguous().cuda()
    start = torch.zeros(2, dtype=torch.int32, device="cuda")
    a = dq.PackedCache(2, 2, 130, 0, 2, 1.99)
    b = dq.PackedCache(2, 2, 130, 0, 2, 1.99)
    dq.quantize_append(a, k, v, start, eye)
    dq.quantize_append(b, k, v, start, None)
    torch.cuda.synchronize()
    for name, t in a.tensors().items():
        assert torch.equal(t, b.tensors()[name]), name


def _bf16_groups_on_thresholds(n_groups, bits, seed):
    """bf16 value groups whose QuEST step Delta has <= 8 significant bits and which
    hold elements exactly on thresholds j*Delta (found by a seeded search, oracle side:
    each threshold replaces the element nearest to it, so Delta barely moves)."""
    rng = np.random.default_rng(seed)
    alpha = QUEST_ALPHA[bits]
    half = 1 << (bits - 1)
    out = []
    for _ in range(200 * n_groups):
        if len(out) == n_groups:
            break
        g = torch.from_numpy(rng.standard_normal(128).astype(np.float32)).bfloat16().float().numpy()
        d = float(orc.quest_meta(g.astype(np.float64), bits, alpha))
        mant = np.frexp(d)[0] * 2 ** 8
        if d == 0 or mant != np.round(mant):          # Delta must be a bf16 value
            continue
        for j in range(-(half - 1), half):
            t = np.float32(j * d)
            if float(torch.tensor([t]).bfloat16().float()[0]) == t:   # only bf16 thresholds
                g[np.argmin(np.abs(g - t))] = t
        if float(orc.quest_meta(g.astype(np.float64), bits, alpha)) == d:
            out.append(g)
    assert len(out) == n_groups
    return np.stack(out)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bf16_values_on_thresholds_bitexact(bits):
    """Values (bf16, no transform) lying exactly on decision thresholds j*Delta take the
    single-product path of the tensor-core append; codes must equal the oracle's."""
    bsz, n, hkv = 1, 256, 1
    v = _bf16_groups_on_thresholds(n, bits, seed=90 + bits).reshape(bsz, n, hkv, 128)
    d = orc.fp16_value(np.array([orc.fp16_bits(orc.quest_meta(g.astype(np.float64), bits, QUEST_ALPHA[bits]))
                                 for g in v.reshape(-1, 128)]))
    ties = sum(int(np.isin(g, [j * dd for j in range(-(1 << (bits - 1)), 1 << (bits - 1))]).sum())
               for g, dd in zip(v.reshape(-1, 128), d))
    assert ties >= n                                   # the test really exercises ties
    k = torch.from_numpy(v.copy()).bfloat16()
    vt = torch.from_numpy(v).bfloat16()
    oc, ost, gc, gst = _run_both(k, vt, orc.QUEST_INT, bits, [0], n)
    assert ost == 0 and gst == 0
    for name in ("v_meta", "v_codes", "k_meta", "k_codes"):
        bad = np.argwhere(oc[name] != gc[name])
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:3].tolist()}"


@pytest.mark.parametrize("kind,bits", CASES)
@pytest.mark.parametrize("bsz,n", [(16, 1), (4, 16)])
def test_small_append_end_to_end(kind, bits, bsz, n):
    """Decode-step sized appends (<= 64 rows) take the one-warp-per-group kernel: same
    bar as the bulk path (value codes/meta bit-exact; key rules as above)."""
    w = QWEN8B_DECODE
    hkv, cap = 2, 48
    start = [(7 * b) % 30 for b in range(bsz)]
    tk = torch.from_numpy(gen.transforms(w)[0][:hkv].copy())
    k = gen.keys(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    _e2e_check(k, v, tk, kind, bits, start, cap)


def test_small_append_capacity_and_status():
    """Rows past the capacity are skipped with status bit 1 on the small path too."""
    w = QWEN8B_DECODE
    k = gen.keys(w, 0, 3, [0, 0, 0], 1)[:, :, :1].contiguous()
    v = gen.values(w, 0, 3, [0, 0, 0], 1)[:, :, :1].contiguous()
    tk = torch.from_numpy(gen.transforms(w)[0][:1].copy())
    oc, ost, gc, gst = _run_both(k, v, 1, 2, [5, 9, 2], 9, tk=tk)       # sequence 1 writes position 9 = cap
    assert ost & orc.STATUS_CAPACITY and gst & dq.STATUS_CAPACITY
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    np.testing.assert_array_equal(oc["v_meta"], gc["v_meta"])
