"""Pins of the CPU oracle to facts outside itself.

Each check takes the oracle module and raises AssertionError on a mismatch.  They
compare the oracle with exact rational arithmetic (fractions), with brute-force
enumeration on tiny inputs, with closed forms and invariants, and with hand-derived
fixtures.  test_oracle_pins runs them on the oracle; test_oracle_mutants plants
plausible mistakes in the oracle and checks that some pin catches each one.
"""
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np

from synth import gen
from synth.configs import QUEST_ALPHA

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
INF = float("inf")


# --------------------------------------------------------------- exact references
def exact_fp16_round(v):
    """Nearest fp16 value (ties to even) of a rational, or +-inf on overflow."""
    v = Fraction(v)
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** (max(e, -14) - 10)
    n = a / q
    fl = n.numerator // n.denominator
    r = n - fl
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    val = fl * q
    if val > 65504:
        return sign * INF
    return sign * val


def _as_float(v):
    return float(v) if not isinstance(v, float) else v


def bits_of_lsb_first(byts, bits):
    """Codes from packed bytes by walking the LSB-first bit string one bit at a time."""
    codes = []
    n_codes = len(byts) * 8 // bits
    for i in range(n_codes):
        c = 0
        for k in range(bits):
            n = bits * i + k
            c |= ((int(byts[n // 8]) >> (n % 8)) & 1) << k
        codes.append(c)
    return codes


# ----------------------------------------------------------------------------- fp16
def check_fp16_rounding(orc):
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(300) * np.exp(rng.uniform(-25, 12, 300)))
    # midpoints between neighbouring fp16 numbers, and one ulp of fp64 either side
    for base in [1.0, 1.5, 3.0, 1000.0, 2.0 ** -14, 2.0 ** -20, 60000.0]:
        h = np.float16(base)
        nxt = np.nextafter(h, np.float16(np.inf))
        mid = (float(h) + float(nxt)) / 2
        vals += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), -mid]
    vals += [65504.0, 65519.99, 65520.0, 70000.0, 2.0 ** -25, 2.0 ** -26, 3 * 2.0 ** -26, 0.0]
    vals = np.array(vals, dtype=np.float64)
    got = orc.fp16_round(vals)
    for v, g in zip(vals, got):
        e = exact_fp16_round(Fraction(float(v)))
        e = e if isinstance(e, float) else float(e)
        assert g == e, (v, g, e)
    # the library conversion numpy float64 -> float16 is correctly rounded as well
    with np.errstate(over="ignore"):
        lib = vals.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(got, lib)


# ------------------------------------------------------------------- QuEST grid
def _quest_groups():
    x = gen.fp32_groups((24, 128), seed=31).numpy().astype(np.float64)
    # constant-magnitude group, a ramp, and a group with values exactly on thresholds
    x[0] = np.where(np.arange(128) % 2 == 0, 0.75, -0.75)
    x[1] = np.arange(128) - 63.5
    return x


def check_quest_step(orc):
    x = _quest_groups()
    getcontext().prec = 60
    for bits in (2, 3, 4):
        alpha = QUEST_ALPHA[bits]
        got = orc.quest_meta(x, bits, alpha)
        for gi in range(x.shape[0]):
            s = sum(Fraction(float(v)) ** 2 for v in x[gi])
            rms = (Decimal(s.numerator) / Decimal(s.denominator) / Decimal(128)).sqrt()
            pre = Decimal(Fraction(alpha).numerator) / Decimal(Fraction(alpha).denominator) * rms
            pre = Fraction(pre) * Fraction(2) ** (1 - bits)
            assert got[gi] == _as_float(exact_fp16_round(pre)), (bits, gi)
    # closed form: every |x| = 0.75 -> RMS = 0.75
    for bits in (2, 3, 4):
        d = orc.quest_meta(x[:1], bits, QUEST_ALPHA[bits])[0]
        assert d == float(exact_fp16_round(Fraction(QUEST_ALPHA[bits]) * Fraction(3, 4)
                                           * Fraction(2) ** (1 - bits)))


def check_quest_codes_bruteforce(orc):
    x = _quest_groups()
    for bits in (2, 3, 4):
        delta = orc.quest_meta(x, bits, QUEST_ALPHA[bits])
        # put some values exactly on thresholds j*Delta and one fp64 ulp either side
        xx = x.copy()
        half = 1 << (bits - 1)
        for gi in range(2, 10):
            for k, j in enumerate(range(-(half - 1), half)):
                xx[gi, 3 * k] = j * delta[gi]
                xx[gi, 3 * k + 1] = np.nextafter(j * delta[gi], -np.inf)
                xx[gi, 3 * k + 2] = np.nextafter(j * delta[gi], np.inf)
        codes = orc.quest_codes(xx, delta, bits)
        for gi in range(xx.shape[0]):
            d = Fraction(float(delta[gi]))
            for i in range(128):
                v = Fraction(float(xx[gi, i]))
                best = None
                for c in range(1 << bits):
                    err = abs(v - (c - half + Fraction(1, 2)) * d)
                    if best is None or err <= best[0]:   # ties go to the upper code
                        best = (err, c)
                assert codes[gi, i] == best[1], (bits, gi, i, float(v), codes[gi, i], best[1])
        deq = orc.quest_dequant(codes, delta, bits)
        inside = (xx >= -half * delta[:, None]) & (xx < half * delta[:, None])
        assert np.all(np.abs(xx - deq)[inside] <= (delta[:, None] / 2 + 0 * xx)[inside])


def check_quest_degenerate(orc):
    x = np.zeros((2, 128))
    for bits in (2, 3, 4):
        d = orc.quest_meta(x, bits, QUEST_ALPHA[bits])
        assert np.all(d == 0.0)
        assert np.all(orc.quest_codes(x, d, bits) == 1 << (bits - 1))
        assert np.all(orc.quest_dequant(orc.quest_codes(x, d, bits), d, bits) == 0.0)


# ---------------------------------------------------------------- percentile affine
def check_affine_bruteforce(orc):
    x = gen.fp32_groups((12, 128), seed=41).numpy().astype(np.float64)
    x[0, :] = np.linspace(-3, 3, 128).astype(np.float32)
    for bits in (2, 3, 4):
        levels = (1 << bits) - 1
        scale, zero = orc.affine_meta(x, bits, 2, 125)
        xx = x.copy()
        for gi in range(1, 6):       # values exactly on the half-way points
            for j in range(levels):
                t = zero[gi] + (j + 0.5) * scale[gi]
                xx[gi, 5 + j] = np.float32(t) if float(np.float32(t)) == t else xx[gi, 5 + j]
        codes = orc.affine_codes(xx, scale, zero, bits)
        for gi in range(x.shape[0]):
            srt = sorted(Fraction(float(v)) for v in x[gi])
            lo, hi = srt[2], srt[125]
            e_scale = exact_fp16_round((hi - lo) / levels)
            e_zero = exact_fp16_round(lo)
            assert scale[gi] == float(e_scale) and zero[gi] == float(e_zero), (bits, gi)
            for i in range(128):
                v = Fraction(float(xx[gi, i]))
                best = None
                for c in range(levels + 1):
                    err = abs(v - (e_zero + c * e_scale))
                    if best is None or err < best[0] or (err == best[0] and c % 2 == 0):
                        best = (err, c)
                assert codes[gi, i] == best[1], (bits, gi, i, float(v))
        deq = orc.affine_dequant(codes, scale, zero)
        inside = (xx >= zero[:, None]) & (xx <= (zero + levels * scale)[:, None])
        assert np.all((np.abs(xx - deq) <= scale[:, None] / 2)[inside])


def check_affine_degenerate(orc):
    x = np.full((1, 128), 1.25)
    s, z = orc.affine_meta(x, 2, 2, 125)
    assert s[0] == 0.0 and z[0] == 1.25
    assert np.all(orc.affine_codes(x, s, z, 2) == 0)
    assert np.all(orc.affine_dequant(orc.affine_codes(x, s, z, 2), s, z) == 1.25)


# ------------------------------------------------------------------------ packing
def check_pack_golden(orc):
    with open(os.path.join(GOLDEN, "pack_ramp.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for bits_s, hexs in rows:
        bits = int(bits_s)
        codes = (np.arange(128) % (1 << bits)).astype(np.uint8)
        period = bytes.fromhex(hexs)
        expect = (period * (16 * bits // len(period) + 1))[: 16 * bits]
        got = orc.pack_codes(codes[None], bits)[0]
        assert bytes(got.tobytes()) == expect, bits
    rng = np.random.default_rng(3)
    for bits in (2, 3, 4):
        c = rng.integers(0, 1 << bits, size=(5, 128)).astype(np.uint8)
        p = orc.pack_codes(c, bits)
        assert p.shape == (5, 16 * bits)
        np.testing.assert_array_equal(orc.unpack_codes(p, bits), c)
        for r in range(5):
            assert bits_of_lsb_first(p[r], bits) == list(c[r])


# ---------------------------------------------------------------------- transform
def check_transform(orc):
    rng = np.random.default_rng(5)
    k = rng.standard_normal((3, 2, 2, 128)).astype(np.float32).astype(np.float64)
    eye = np.stack([np.eye(128)] * 2)
    np.testing.assert_array_equal(orc.transform_keys(k, eye), k)
    t, tinv = gen.key_transform_pair(np.random.default_rng(9))
    t32 = np.stack([t.astype(np.float32).astype(np.float64), np.eye(128)[::-1]])
    x = orc.transform_keys(k, t32)
    for (a, b, h) in [(0, 0, 0), (2, 1, 0), (1, 0, 1)]:
        for i in (0, 5, 127):
            ex = sum(Fraction(float(t32[h, i, j])) * Fraction(float(k[a, b, h, j]))
                     for j in range(128))
            assert abs(x[a, b, h, i] - float(ex)) <= 1e-13 * (1 + abs(float(ex))), (a, b, h, i)
    # T_k^{-T} from the closed form is the numeric inverse-transpose; orthogonal T maps to itself
    np.testing.assert_allclose(tinv, np.linalg.inv(t).T, atol=1e-12)
    q = gen.haar_orthogonal(np.random.default_rng(4))
    np.testing.assert_allclose(np.linalg.inv(q).T, q, atol=1e-12)
    # query map: head h uses KV head h // g
    qq = rng.standard_normal((2, 4, 128))
    m = np.stack([t, np.eye(128)])
    out = orc.transform_query(qq, m, 2)
    for b in range(2):
        for h in range(4):
            ex = m[h // 2] @ qq[b, h]
            np.testing.assert_allclose(out[b, h], ex, rtol=1e-12, atol=1e-12)


def check_unquantized_invariance(orc):
    """(T^{-T} q) . (T k) = q . k: attention with transformed queries and keys
    equals attention on the originals."""
    rng = np.random.default_rng(11)
    t, tinv = gen.key_transform_pair(rng)
    k = rng.standard_normal((1, 64, 1, 128)) * 3
    q = rng.standard_normal((1, 4, 128))
    x = orc.transform_keys(k, t[None])[0, :, 0, :]
    qt = orc.transform_query(q, tinv[None], 1)[0]
    s1 = qt @ x.T
    s0 = q[0] @ k[0, :, 0, :].T
    np.testing.assert_allclose(s1, s0, rtol=1e-10, atol=1e-10)


# ----------------------------------------------------------------------- attention
def _small_cache(orc, kind, bits, ctx=40, batch=2, hkv=2):
    rng = np.random.default_rng(21)
    cache = orc.empty_cache(batch, hkv, ctx + 8, kind, bits)
    k = rng.standard_normal((batch, ctx, hkv, 128)) * np.exp(rng.standard_normal(128))
    v = rng.standard_normal((batch, ctx, hkv, 128))
    alpha = QUEST_ALPHA.get(bits, 2.0)
    st = orc.quantize_append(cache, k.astype(np.float32), v.astype(np.float32),
                             [0] * batch, kind, bits, alpha, 2, 125)
    assert st == 0
    return cache


def check_decode_bruteforce(orc):
    for kind, bits in ((0, 2), (1, 2), (0, 3), (1, 4)):
        cache = _small_cache(orc, kind, bits)
        rng = np.random.default_rng(23)
        hq, hkv = 4, 2
        q = rng.standard_normal((2, hq, 128))
        ctx = [40, 17]
        tau = 1 / math.sqrt(128)
        got = orc.decode_attention(cache, q, ctx, tau, kind, bits, hkv)
        half = 1 << (bits - 1)
        for b in range(2):
            for h in range(hq):
                kv = h // (hq // hkv)
                kh, vh = [], []
                for side, dst in (("k", kh), ("v", vh)):
                    for t in range(ctx[b]):
                        codes = bits_of_lsb_first(cache[f"{side}_codes"][b, kv, t], bits)
                        meta = [float(np.uint16(m).view(np.float16))
                                for m in cache[f"{side}_meta"][b, kv, t]]
                        if kind == 0:
                            dst.append([(c - half + 0.5) * meta[0] for c in codes])
                        else:
                            dst.append([meta[1] + c * meta[0] for c in codes])
                s = [tau * sum(q[b, h, i] * kh[t][i] for i in range(128)) for t in range(ctx[b])]
                mx = max(s)
                p = [math.exp(v - mx) for v in s]
                den = sum(p)
                o = [sum(p[t] * vh[t][i] for t in range(ctx[b])) / den for i in range(128)]
                np.testing.assert_allclose(got[b, h], o, rtol=1e-10, atol=1e-10)


def check_decode_special(orc):
    kind, bits = 1, 2
    cache = _small_cache(orc, kind, bits)
    rng = np.random.default_rng(29)
    q = rng.standard_normal((2, 4, 128))
    tau = 1 / math.sqrt(128)
    # ctx_len 1: output is the first dequantized value row; ctx_len 0: zeros
    out = orc.decode_attention(cache, q, [1, 0], tau, kind, bits, 2)
    v0 = orc.dequant_groups(orc.unpack_codes(cache["v_codes"][0, :, 0], bits),
                            cache["v_meta"][0, :, 0], kind, bits)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], v0[h // 2], rtol=1e-14, atol=1e-14)
    assert np.all(out[1] == 0)
    # identical keys: uniform weights, output is the mean of the value rows
    c2 = {k: v.copy() for k, v in cache.items()}
    c2["k_codes"][:] = c2["k_codes"][:, :, :1]
    c2["k_meta"][:] = c2["k_meta"][:, :, :1]
    out = orc.decode_attention(c2, q, [40, 17], tau, kind, bits, 2)
    for b, n in ((0, 40), (1, 17)):
        vh = orc.dequant_groups(orc.unpack_codes(cache["v_codes"][b, :, :n], bits),
                                cache["v_meta"][b, :, :n], kind, bits)
        for h in range(4):
            np.testing.assert_allclose(out[b, h], vh[h // 2].mean(axis=0), rtol=1e-12, atol=1e-12)


def check_chunk_bruteforce(orc):
    """Chunk attention (R18) against per-query windows written out by hand: query i of
    a chunk of n_q sees positions 0 .. ctx - n_q + i of its KV head."""
    kind, bits = 0, 2
    cache = _small_cache(orc, kind, bits, ctx=12)
    rng = np.random.default_rng(31)
    hq, hkv, nq = 4, 2, 5
    q = rng.standard_normal((2, nq, hq, 128))
    ctx = [12, 3]                      # sequence 1: the first two queries precede position 0
    tau = 1 / math.sqrt(128)
    got = orc.chunk_attention(cache, q, ctx, tau, kind, bits, hkv)
    half = 1 << (bits - 1)
    for b in range(2):
        for kv in range(hkv):
            kh, vh = [], []
            for side, dst in (("k", kh), ("v", vh)):
                for t in range(ctx[b]):
                    codes = bits_of_lsb_first(cache[f"{side}_codes"][b, kv, t], bits)
                    delta = float(np.uint16(cache[f"{side}_meta"][b, kv, t, 0]).view(np.float16))
                    dst.append([(c - half + 0.5) * delta for c in codes])
            for i in range(nq):
                last = ctx[b] - nq + i          # the query's own position
                for h in range(kv * 2, kv * 2 + 2):
                    if last < 0:
                        assert np.all(got[b, i, h] == 0)
                        continue
                    s = [tau * sum(q[b, i, h, c] * kh[t][c] for c in range(128)) for t in range(last + 1)]
                    mx = max(s)
                    p = [math.exp(v - mx) for v in s]
                    den = sum(p)
                    o = [sum(p[t] * vh[t][c] for t in range(last + 1)) / den for c in range(128)]
                    np.testing.assert_allclose(got[b, i, h], o, rtol=1e-10, atol=1e-10)


def check_chunk_special(orc):
    """Chunk attention invariants: its last query is the decode query at the same
    context (decode is pinned by brute force above); a query cannot see the positions
    after its own; a chunk query at position 0 returns the first value row."""
    kind, bits = 1, 3
    cache = _small_cache(orc, kind, bits)
    rng = np.random.default_rng(37)
    hq, hkv, nq = 4, 2, 16
    q = rng.standard_normal((2, nq, hq, 128))
    tau = 1 / math.sqrt(128)
    ctx = [40, 17]
    out = orc.chunk_attention(cache, q, ctx, tau, kind, bits, hkv)
    dec = orc.decode_attention(cache, q[:, nq - 1], ctx, tau, kind, bits, hkv)
    np.testing.assert_allclose(out[:, nq - 1], dec, rtol=1e-13, atol=1e-13)
    # sequence 0: query i sits at position 24 + i.  Overwrite positions 32 .. 39 (those
    # of queries 8 .. 15): queries 0..7 keep their outputs, queries 8 onwards change.
    first = 40 - nq + 8
    c2 = {k: v.copy() for k, v in cache.items()}
    c2["k_codes"][0, :, first:40] ^= 0x5A
    c2["v_codes"][0, :, first:40] ^= 0x3C
    out2 = orc.chunk_attention(c2, q, ctx, tau, kind, bits, hkv)
    assert np.array_equal(out2[0, :8], out[0, :8])
    assert np.array_equal(out2[1], out[1])
    for i in range(8, nq):
        assert not np.allclose(out2[0, i], out[0, i]), i
    # sequence of 16 tokens, chunk of 16: query 0 sees position 0 only
    out3 = orc.chunk_attention(cache, q, [nq, nq], tau, kind, bits, hkv)
    for b in range(2):
        v0 = orc.dequant_groups(orc.unpack_codes(cache["v_codes"][b, :, 0], bits),
                                cache["v_meta"][b, :, 0], kind, bits)
        for h in range(hq):
            np.testing.assert_allclose(out3[b, 0, h], v0[h // 2], rtol=1e-14, atol=1e-14)


def check_rope(orc):
    """RoPE (R19): identity at angle 0; a quarter turn maps the pair (x, y) of channels
    (i, i + 64) to (-y, x); the rotation keeps the norm; rotated dot products depend only
    on the difference of the positions (table built here from math.cos / math.sin)."""
    rng = np.random.default_rng(41)
    k = rng.standard_normal((3, 128))
    assert np.array_equal(orc.apply_rope(k, np.ones(64), np.zeros(64)), k)
    for i in (0, 17, 63):
        e = np.zeros(128)
        e[i] = 1.0
        cos, sin = np.zeros(64), np.zeros(64)
        cos[:] = 1.0
        cos[i], sin[i] = 0.0, 1.0                     # quarter turn of pair i only
        out = orc.apply_rope(e, cos, sin)
        want = np.zeros(128)
        want[i + 64] = 1.0
        assert np.array_equal(out, want), i
        e2 = np.zeros(128)
        e2[i + 64] = 1.0
        want2 = np.zeros(128)
        want2[i] = -1.0
        assert np.array_equal(orc.apply_rope(e2, cos, sin), want2), i

    def table_row(p, theta=1.0e6):
        ang = [p * theta ** (-2.0 * j / 128) for j in range(64)]
        return np.array([math.cos(a) for a in ang]), np.array([math.sin(a) for a in ang])
    q = rng.standard_normal(128)
    c5, s5 = table_row(5)
    c2, s2 = table_row(2)
    c13, s13 = table_row(13)
    c10, s10 = table_row(10)
    rq = orc.apply_rope(q, c5, s5)
    np.testing.assert_allclose(np.linalg.norm(rq), np.linalg.norm(q), rtol=1e-14)
    d1 = rq @ orc.apply_rope(k[0], c2, s2)
    d2 = orc.apply_rope(q, c13, s13) @ orc.apply_rope(k[0], c10, s10)
    np.testing.assert_allclose(d1, d2, rtol=1e-11, atol=1e-11)
    assert abs(d1 - q @ k[0]) > 1e-3                  # the rotation does change the product


def check_append_rope(orc):
    """Fused-RoPE append (R19): an identity table gives the plain append; a table that
    turns only position 5 by a quarter turn changes only the row written at position 5,
    and that row equals the plain append of the key with its pairs swapped as (-y, x)."""
    rng = np.random.default_rng(43)
    bsz, n, hkv, cap = 2, 4, 2, 12
    k = rng.standard_normal((bsz, n, hkv, 128)) * np.exp(rng.standard_normal(128))
    v = rng.standard_normal((bsz, n, hkv, 128))
    tk = np.stack([np.linalg.qr(rng.standard_normal((128, 128)))[0] for _ in range(hkv)])
    start = [3, 8]                                    # sequence 0 writes positions 3..6, sequence 1 8..11
    ident = np.concatenate([np.ones((cap, 64)), np.zeros((cap, 64))], axis=1)
    for kind, bits, alpha in ((0, 2, QUEST_ALPHA[2]), (1, 3, 0.0)):
        a = orc.empty_cache(bsz, hkv, cap, kind, bits)
        b = orc.empty_cache(bsz, hkv, cap, kind, bits)
        assert orc.quantize_append_rope(a, k, v, start, ident, kind, bits, alpha, tk=tk) == 0
        assert orc.quantize_append(b, k, v, start, kind, bits, alpha, tk=tk) == 0
        for name in a:
            assert np.array_equal(a[name], b[name]), name
        quarter = ident.copy()
        quarter[5] = np.concatenate([np.zeros(64), np.ones(64)])
        c = orc.empty_cache(bsz, hkv, cap, kind, bits)
        assert orc.quantize_append_rope(c, k, v, start, quarter, kind, bits, alpha, tk=tk) == 0
        swapped = k.copy()
        swapped[0, 2] = np.concatenate([-k[0, 2, :, 64:], k[0, 2, :, :64]], axis=-1)   # position 3 + 2 = 5
        d = orc.empty_cache(bsz, hkv, cap, kind, bits)
        assert orc.quantize_append(d, swapped, v, start, kind, bits, alpha, tk=tk) == 0
        for name in c:
            assert np.array_equal(c[name], d[name]), name
        assert not np.array_equal(c["k_codes"][0, :, 5], a["k_codes"][0, :, 5])
        assert np.array_equal(c["v_codes"], a["v_codes"])


def check_structured_transforms(orc):
    """Structured key transforms (R20): the Sylvester Hadamard matrix equals the library's
    (scipy.linalg.hadamard) and H H^T = n I; the closed-form inverse-transpose of
    H diag(s) / sqrt(128) equals numpy's inverse, and keeps q' . x = q . k; a
    block-diagonal T_k applied to keys equals the per-block products written as loops."""
    import scipy.linalg
    for n in (1, 2, 8, 128):
        h = orc.hadamard(n)
        assert np.array_equal(h, scipy.linalg.hadamard(n).astype(np.float64)), n
        assert np.array_equal(h @ h.T, n * np.eye(n)), n
    rng = np.random.default_rng(47)
    s = np.exp(rng.uniform(np.log(0.25), np.log(4.0), (2, 128))) * rng.choice([-1.0, 1.0], (2, 128))
    t = orc.hadamard_diag_transform(s)
    m = orc.hadamard_diag_inverse_transpose(s)
    for i in range(2):
        np.testing.assert_allclose(m[i], np.linalg.inv(t[i]).T, rtol=1e-12, atol=1e-13)
    k = rng.standard_normal((3, 2, 128))
    q = rng.standard_normal((3, 2, 128))
    x = orc.transform_keys(k, t)
    qt = orc.transform_query(q, m, 2)
    np.testing.assert_allclose(np.sum(qt * x, axis=-1), np.sum(q * k, axis=-1), rtol=1e-11, atol=1e-11)
    for bs in (16, 32, 64):
        blocks = rng.standard_normal((2, 128 // bs, bs, bs))
        tk = orc.block_diagonal_transform(blocks)
        got = orc.transform_keys(k, tk)
        for a in range(3):
            for h in range(2):
                for j in range(128 // bs):
                    for r in range(bs):
                        want = sum(blocks[h, j, r, c] * k[a, h, j * bs + c] for c in range(bs))
                        assert abs(got[a, h, j * bs + r] - want) <= 1e-12 * (1 + abs(want)), (bs, a, h, j, r)


def check_decode_pair(orc):
    """decode_attention_pair (one sequence and KV head, used for sampled full-size checks)
    against an explicit-loop softmax over hand-dequantized rows."""
    kind, bits = 1, 2
    cache = _small_cache(orc, kind, bits, ctx=9, batch=1, hkv=1)
    rng = np.random.default_rng(53)
    q = rng.standard_normal((2, 128))
    tau = 0.125
    n = 7
    got = orc.decode_attention_pair(cache["k_codes"][0, 0, :n], cache["k_meta"][0, 0, :n], cache["v_codes"][0, 0, :n],
                                    cache["v_meta"][0, 0, :n], q, tau, kind, bits)
    rows = {}
    for side in ("k", "v"):
        rows[side] = []
        for t in range(n):
            codes = bits_of_lsb_first(cache[f"{side}_codes"][0, 0, t], bits)
            sc, z = [float(np.uint16(m).view(np.float16)) for m in cache[f"{side}_meta"][0, 0, t]]
            rows[side].append([z + c * sc for c in codes])
    for i in range(2):
        s = [tau * sum(q[i, c] * rows["k"][t][c] for c in range(128)) for t in range(n)]
        mx = max(s)
        p = [math.exp(x - mx) for x in s]
        o = [sum(p[t] * rows["v"][t][c] for t in range(n)) / sum(p) for c in range(128)]
        np.testing.assert_allclose(got[i], o, rtol=1e-10, atol=1e-10)
    empty = orc.decode_attention_pair(cache["k_codes"][0, 0, :0], cache["k_meta"][0, 0, :0], cache["v_codes"][0, 0, :0],
                                      cache["v_meta"][0, 0, :0], q, tau, kind, bits)
    assert np.all(empty == 0)


def check_gather_paged(orc):
    """gather_paged against entries labelled with their page and row: position t of
    sequence b must come from row t % page_size of page block_table[b][t // page_size]."""
    num_pages, hkv, ps = 7, 2, 4
    pool = np.zeros((num_pages, hkv, ps, 3), dtype=np.int64)
    for pg in range(num_pages):
        for h in range(hkv):
            for r in range(ps):
                pool[pg, h, r] = [pg, h, r]
    bt = np.array([[5, 0, 3], [2, 6, 1]])
    out = orc.gather_paged(pool, bt, ps)
    assert out.shape == (2, hkv, 3 * ps, 3)
    for b in range(2):
        for h in range(hkv):
            for t in range(3 * ps):
                assert out[b, h, t].tolist() == [bt[b][t // ps], h, t % ps], (b, h, t)


def check_append_positions(orc):
    cache = orc.empty_cache(2, 1, 10, 0, 2)
    x = np.ones((2, 3, 1, 128))
    x[1] *= -2.0
    st = orc.quantize_append(cache, x, x, [2, 8], 0, 2, 1.99)
    assert st == 1                                   # positions 10 of sequence 1 overflow
    assert np.all(cache["k_codes"][0, 0, 2:5] != 0) and np.all(cache["k_codes"][0, 0, :2] == 0)
    assert np.all(cache["k_codes"][0, 0, 5:] == 0)
    assert np.all(cache["k_meta"][1, 0, 8:10] != 0) and np.all(cache["k_meta"][1, 0, :8] == 0)
    # all-equal positive group: Delta = fp16(1.99 * 0.5) and every code is 2 (x >= 0, x < Delta)
    d = float(exact_fp16_round(Fraction(1.99) / 2))
    assert orc.fp16_value(cache["k_meta"][0, 0, 2, 0]) == d
    assert orc.unpack_codes(cache["k_codes"][0, 0, 2], 2).tolist() == [3 if 1.0 >= d else 2] * 128


ALL_PINS = [
    check_fp16_rounding, check_quest_step, check_quest_codes_bruteforce, check_quest_degenerate,
    check_affine_bruteforce, check_affine_degenerate, check_pack_golden, check_transform,
    check_unquantized_invariance, check_decode_bruteforce, check_decode_special,
    check_chunk_bruteforce, check_chunk_special, check_rope, check_append_rope, check_structured_transforms,
    check_decode_pair, check_gather_paged, check_append_positions,
]

