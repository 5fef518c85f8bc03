"""Plain fp64 CPU oracle of the WUSH-KV runtime hot path.

TEST INFRASTRUCTURE.  Only the tests, the smoke check of the graft entry point and
the benchmark's CPU-baseline / reference legs may import or run this module.  The
product path (the CUDA library and its Python binding) never calls it, and it
shares no code, table or constant generator with that path.

Every function is the plain definition, written out in numpy float64, with no
blocking, fusion or reordering beyond what the definition states.  Sources (the
only material on the method is a handful of web pages about the preprint
"WUSH-KV: KV Cache Quantization with Data-Adaptive Transforms"):

  [ai4s]   ai4snews summary "WUSH-KV cuts 2-bit KV-cache perplexity from OSCAR's
           13.74 to 10.51 ...", paragraphs 1-6.
  [blog]   cere-bro page "WUSH-KV: 2-bit KV-Cache Quantization with Data-Adaptive
           Transforms", sections TL;DR, flowchart, Gaps.
  [abs]    the arXiv abstract (readsearch.ai and searcharxiv listings).

What the pages fix: a per-KV-head key transform applied to post-RoPE keys
([ai4s] paragraphs 1 and 5; [blog] TL;DR; [abs]); values already in the
transformed basis because their transform is folded into the weights ([ai4s]
paragraph 5; [blog] flowchart); a clipped per-token scalar quantizer, QuEST-INT or
OSCAR-style percentile-clipped affine ([ai4s] paragraphs 3-5; [abs]); 2-bit KV
caches served with grouped-query attention ([ai4s] paragraph 5).  What the pages
leave open is taken in its plainest reading; each reading is named where it is
used (R1..R12 and R18..R20 below; R13..R17 concern the input generator and
the parity rules, not the oracle) and listed in the design notes.

Readings:
  R1  x = T_k k with column vectors; T_k stored row-major, x_i = sum_j T_ij k_j.
  R2  the decode query is mapped by M = T_k^{-T} of its KV head, so that
      (M q) . (T_k k) = q . k and attention is unchanged by the key transform.
  R3  QuEST-INT-style grid: RMS = sqrt(sum x^2 / 128); step
      Delta = fp16(alpha * RMS * 2^(1-b)); code = clamp(floor(x/Delta) + 2^(b-1),
      0, 2^b - 1), evaluated as the count of thresholds j*Delta,
      j in [-(2^(b-1)-1), 2^(b-1)-1], with x >= j*Delta; dequant
      (code - 2^(b-1) + 1/2) * Delta.
  R4  percentile affine grid: lo, hi = elements of 0-based ascending rank r_lo,
      r_hi; scale = fp16((hi - lo) / (2^b - 1)) from the unrounded lo, hi;
      zero = fp16(lo); code = clamp(round-half-even((x - zero)/scale), 0, 2^b-1)
      using the stored fp16 scale and zero, evaluated by exact comparisons with
      the thresholds zero + (j + 1/2) scale; dequant zero + code * scale.
  R5  fp16 conversions round to nearest, ties to even, once, straight from fp64.
  R6  degenerate groups: Delta == 0 gives code 2^(b-1) everywhere; scale == 0
      gives code 0 everywhere.
  R7  packing: the 128 codes of a group form one LSB-first bit string, element i
      at bits [b*i, b*i + b); bit n is bit (n mod 8) of byte n // 8.  16*b bytes.
  R8  attention: s_t = tau * q' . k_hat_t over t < ctx_len, softmax with the max
      subtracted, output sum_t p_t v_hat_t in the transformed value basis.
  R9  GQA: query head h reads KV head h // (Hq / Hkv).
  R10 ctx_len == 0 gives an all-zero output row.
  R11 positions >= capacity are not written and set status bit 1.
  R12 the value side uses the same quantizer kind, bits and parameters as the
      key side, on the untransformed value.
  R19 fused RoPE ([ai4s] paragraph 5: the key transform follows RoPE): rotate-half
      pairs (i, i + 64), k_i -> k_i cos_i - k_{i+64} sin_i and k_{i+64} -> k_{i+64}
      cos_i + k_i sin_i for i < 64, with cos, sin read from row p (the key's
      position) of a caller-supplied fp32 table [rows][128] (cos in the first 64
      entries, sin in the last 64); the rotated key is not rounded before the
      transform.
  R20 structured key transforms ([ai4s] paragraph 6: cheaper structured transforms
      are the authors' future work; Hadamard is a baseline): (a) block-diagonal T_k,
      n/b blocks of b x b on the diagonal, block j acting on channels [j b, (j+1) b);
      (b) T_k = H diag(s) / sqrt(128) with H the Sylvester Hadamard matrix
      (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]) and s a per-channel scale.  Both
      are ordinary invertible T_k, applied by the same definition x = T_k k (R1).
  R18 chunked forward ([ai4s] paragraph 3: sequences run in 16-token forward
      chunks): the chunk's n_q tokens are appended to the cache first, then query i
      of the chunk (0-based) sits at position ctx - n_q + i, ctx = min(ctx_len,
      capacity), and attends every cached position up to and including its own,
      all read from the packed cache.  A query whose position is negative gives an
      all-zero row (R10).
"""
import numpy as np

QUEST_INT = 0
PCT_AFFINE = 1
HEAD_DIM = 128

STATUS_CAPACITY = 1
STATUS_NONFINITE = 2
STATUS_META_OVERFLOW = 4
STATUS_CTX_OVER_CAPACITY = 8

FP16_MAX = 65504.0


# ----------------------------------------------------------------------------- fp16
def fp16_round(x):
    """Round float64 values to the nearest fp16 value, ties to even (R5).

    Written from the IEEE 754 binary16 definition: 11 significant bits, minimum
    normal exponent -14, quantum 2^-24 below it, overflow to infinity at or above
    the midpoint 65520 between 65504 and 2^16.  Scaling by powers of two is exact
    in float64, and np.rint rounds half to even.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, e = np.frexp(ax)                       # ax = m * 2**e, m in [0.5, 1)
    lead = e.astype(np.int64) - 1             # exponent of the leading bit
    q_exp = np.maximum(lead, -14) - 10        # exponent of the fp16 quantum
    with np.errstate(invalid="ignore", over="ignore"):
        n = np.rint(np.ldexp(ax, -q_exp))
        r = np.ldexp(n, q_exp)
    r = np.where(ax == 0.0, 0.0, r)
    r = np.where(np.isfinite(ax) & (r > FP16_MAX), np.inf, r)
    return np.copysign(r, x)


def fp16_bits(values):
    """Bit patterns (uint16) of values that are already exact fp16 numbers."""
    v = np.asarray(values, dtype=np.float64)
    h = v.astype(np.float16)
    assert np.array_equal(h.astype(np.float64), v, equal_nan=True), "value not exact in fp16"
    return h.view(np.uint16)


def fp16_value(bits):
    """float64 value of fp16 bit patterns."""
    return np.asarray(bits).astype(np.uint16).view(np.float16).astype(np.float64)


# ------------------------------------------------------------------ key transform
def transform_keys(k, tk):
    """x = T_k k per (token, KV head) (R1).  k: [..., Hkv, 128], tk: [Hkv, 128, 128]."""
    k = np.asarray(k, dtype=np.float64)
    tk = np.asarray(tk, dtype=np.float64)
    x = np.empty_like(k)
    for h in range(tk.shape[0]):
        x[..., h, :] = k[..., h, :] @ tk[h].T
    return x


def block_diagonal_transform(blocks):
    """Dense T_k [Hkv, 128, 128] of block-diagonal transforms (R20a).
    blocks: [Hkv, 128 / b, b, b]; block j sits on rows and columns [j b, (j + 1) b)."""
    blocks = np.asarray(blocks, dtype=np.float64)
    hkv, nb, bs, _ = blocks.shape
    assert nb * bs == HEAD_DIM
    tk = np.zeros((hkv, HEAD_DIM, HEAD_DIM))
    for h in range(hkv):
        for j in range(nb):
            tk[h, j * bs:(j + 1) * bs, j * bs:(j + 1) * bs] = blocks[h, j]
    return tk


def hadamard(n):
    """Sylvester Hadamard matrix of order n (a power of two) (R20b)."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    assert h.shape[0] == n
    return h


def hadamard_diag_transform(scale):
    """T_k = H diag(s) / sqrt(128) per KV head (R20b).  scale: [Hkv, 128], nonzero."""
    s = np.asarray(scale, dtype=np.float64)
    h = hadamard(HEAD_DIM) / np.sqrt(HEAD_DIM)
    return np.stack([h * s[i][None, :] for i in range(s.shape[0])])


def hadamard_diag_inverse_transpose(scale):
    """T_k^{-T} of hadamard_diag_transform: H diag(1/s) / sqrt(128), since H / sqrt(128)
    is symmetric and orthogonal (R2, R20b)."""
    s = np.asarray(scale, dtype=np.float64)
    h = hadamard(HEAD_DIM) / np.sqrt(HEAD_DIM)
    return np.stack([h / s[i][None, :] for i in range(s.shape[0])])


def transform_query(q, tk_inv_t, num_kv_heads):
    """q' = T_k^{-T} q with the KV head of each query head's group (R2, R9).
    q: [B, Hq, 128]; tk_inv_t: [Hkv, 128, 128]."""
    q = np.asarray(q, dtype=np.float64)
    m = np.asarray(tk_inv_t, dtype=np.float64)
    g = q.shape[1] // num_kv_heads
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        out[:, h, :] = q[:, h, :] @ m[h // g].T
    return out


# --------------------------------------------------------------------- quantizers
def quest_step_prerounding(x, bits, alpha):
    """alpha * RMS * 2^(1-b) in float64 before the fp16 rounding (R3)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.sum(x * x, axis=-1)
    rms = np.sqrt(s / HEAD_DIM)
    return alpha * rms * 2.0 ** (1 - bits)


def quest_meta(x, bits, alpha):
    """fp16 step Delta per group (value, float64) (R3, R5)."""
    return fp16_round(quest_step_prerounding(x, bits, alpha))


def quest_codes(x, delta, bits):
    """Codes by counting the thresholds j*Delta that x reaches (R3, R6)."""
    x = np.asarray(x, dtype=np.float64)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    half = 1 << (bits - 1)
    codes = np.zeros(x.shape, dtype=np.uint8)
    for j in range(-(half - 1), half):
        codes += (x >= j * d).astype(np.uint8)
    return np.where(d == 0.0, np.uint8(half), codes).astype(np.uint8)


def quest_dequant(codes, delta, bits):
    half = 1 << (bits - 1)
    return (np.asarray(codes, np.float64) - half + 0.5) * np.asarray(delta, np.float64)[..., None]


def affine_prerounding(x, bits, rank_lo, rank_hi):
    """(scale before rounding, lo) of the percentile affine grid (R4)."""
    x = np.asarray(x, dtype=np.float64)
    part = np.partition(x, (rank_lo, rank_hi), axis=-1)
    lo = part[..., rank_lo]
    hi = part[..., rank_hi]
    return (hi - lo) / ((1 << bits) - 1), lo


def affine_meta(x, bits, rank_lo, rank_hi):
    """fp16 (scale, zero) per group as float64 values (R4, R5)."""
    scale_pre, lo = affine_prerounding(x, bits, rank_lo, rank_hi)
    return fp16_round(scale_pre), fp16_round(lo)


def affine_codes(x, scale, zero, bits):
    """round-half-even((x - zero)/scale) clamped, by exact threshold comparisons (R4, R6).

    zero + (j + 1/2) * scale is exact in float64: both terms are multiples of 2^-25
    below 2^17, and x is an fp32 or bf16 value, so every comparison is exact.
    """
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float64)[..., None]
    z = np.asarray(zero, dtype=np.float64)[..., None]
    codes = np.zeros(x.shape, dtype=np.uint8)
    for j in range((1 << bits) - 1):
        t = z + (j + 0.5) * s
        up = (x > t) | ((x == t) & (j % 2 == 1))
        codes += up.astype(np.uint8)
    return np.where(s == 0.0, np.uint8(0), codes).astype(np.uint8)


def affine_dequant(codes, scale, zero):
    return (np.asarray(zero, np.float64)[..., None]
            + np.asarray(codes, np.float64) * np.asarray(scale, np.float64)[..., None])


def quantize_groups(x, kind, bits, clip_alpha=0.0, rank_lo=2, rank_hi=125):
    """Codes [..., 128] (uint8) and meta [..., m] (fp16 bit patterns, uint16)."""
    if kind == QUEST_INT:
        delta = quest_meta(x, bits, clip_alpha)
        return quest_codes(x, delta, bits), fp16_bits(delta)[..., None]
    if kind == PCT_AFFINE:
        scale, zero = affine_meta(x, bits, rank_lo, rank_hi)
        codes = affine_codes(x, scale, zero, bits)
        return codes, np.stack([fp16_bits(scale), fp16_bits(zero)], axis=-1)
    raise ValueError(kind)


def dequant_groups(codes, meta_bits, kind, bits):
    meta = fp16_value(meta_bits)
    if kind == QUEST_INT:
        return quest_dequant(codes, meta[..., 0], bits)
    return affine_dequant(codes, meta[..., 0], meta[..., 1])


# ------------------------------------------------------------------------ packing
def pack_codes(codes, bits):
    """LSB-first bit string of each 128-code group (R7): [..., 128] -> [..., 16*bits]."""
    c = np.asarray(codes, dtype=np.uint8)
    planes = (c[..., :, None] >> np.arange(bits, dtype=np.uint8)) & 1
    flat = planes.reshape(c.shape[:-1] + (c.shape[-1] * bits,))
    return np.packbits(flat, axis=-1, bitorder="little")


def unpack_codes(packed, bits):
    p = np.asarray(packed, dtype=np.uint8)
    flat = np.unpackbits(p, axis=-1, bitorder="little")
    planes = flat.reshape(p.shape[:-1] + (p.shape[-1] * 8 // bits, bits)).astype(np.uint8)
    return np.sum(planes << np.arange(bits, dtype=np.uint8), axis=-1).astype(np.uint8)


# ------------------------------------------------------------------ cache + append
def empty_cache(batch, num_kv_heads, capacity, kind, bits):
    m = 1 if kind == QUEST_INT else 2
    return {
        "k_codes": np.zeros((batch, num_kv_heads, capacity, 16 * bits), np.uint8),
        "v_codes": np.zeros((batch, num_kv_heads, capacity, 16 * bits), np.uint8),
        "k_meta": np.zeros((batch, num_kv_heads, capacity, m), np.uint16),
        "v_meta": np.zeros((batch, num_kv_heads, capacity, m), np.uint16),
    }


def quantize_append(cache, k_new, v_new, start_pos, kind, bits, clip_alpha=0.0,
                    rank_lo=2, rank_hi=125, tk=None):
    """Transform (unless tk is None), quantize and pack K and V, then write them at
    positions start_pos[b] .. start_pos[b] + n - 1 of each sequence (R1, R3, R4, R7,
    R11, R12).  k_new, v_new: [B, n, Hkv, 128] real values.  Returns the status bits."""
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    x = transform_keys(k_new, tk) if tk is not None else k_new
    cap = cache["k_codes"].shape[2]
    status = 0
    if not (np.all(np.isfinite(k_new)) and np.all(np.isfinite(v_new))):
        status |= STATUS_NONFINITE
    for side, vals in (("k", x), ("v", v_new)):
        codes, meta = quantize_groups(vals, kind, bits, clip_alpha, rank_lo, rank_hi)
        if np.any(~np.isfinite(fp16_value(meta))):
            status |= STATUS_META_OVERFLOW
        packed = pack_codes(codes, bits)                      # [B, n, Hkv, 16b]
        for b in range(vals.shape[0]):
            for t in range(vals.shape[1]):
                pos = int(start_pos[b]) + t
                if pos < 0 or pos >= cap:
                    status |= STATUS_CAPACITY
                    continue
                cache[f"{side}_codes"][b, :, pos, :] = packed[b, t]
                cache[f"{side}_meta"][b, :, pos, :] = meta[b, t]
    return status


# ---------------------------------------------------------------------------- RoPE
def apply_rope(k, cos, sin):
    """Rotate-half RoPE (R19): k [..., 128]; cos, sin [..., 64] broadcast against it."""
    k = np.asarray(k, dtype=np.float64)
    cos = np.asarray(cos, dtype=np.float64)
    sin = np.asarray(sin, dtype=np.float64)
    lo, hi = k[..., :HEAD_DIM // 2], k[..., HEAD_DIM // 2:]
    return np.concatenate([lo * cos - hi * sin, hi * cos + lo * sin], axis=-1)


def quantize_append_rope(cache, k_pre, v_new, start_pos, rope_table, kind, bits, clip_alpha=0.0,
                         rank_lo=2, rank_hi=125, tk=None):
    """RoPE fused in front of the transform (R19): the key of position p = start_pos[b] + t
    is rotated with row p of rope_table [rows >= capacity][128], then appended exactly as
    quantize_append does.  k_pre: [B, n, Hkv, 128] pre-RoPE keys."""
    k_pre = np.asarray(k_pre, dtype=np.float64)
    tab = np.asarray(rope_table, dtype=np.float64)
    capacity = cache["k_codes"].shape[2]
    assert tab.shape[0] >= capacity and tab.shape[1] == HEAD_DIM
    bsz, n = k_pre.shape[:2]
    k_rot = k_pre.copy()
    for b in range(bsz):
        for t in range(n):
            p = int(start_pos[b]) + t
            if 0 <= p < capacity:             # other positions are not written (R11)
                k_rot[b, t] = apply_rope(k_pre[b, t], tab[p, :HEAD_DIM // 2], tab[p, HEAD_DIM // 2:])
    return quantize_append(cache, k_rot, v_new, start_pos, kind, bits, clip_alpha, rank_lo, rank_hi, tk=tk)


# ----------------------------------------------------------------------- attention
def decode_attention(cache, q_t, ctx_len, softmax_scale, kind, bits, num_kv_heads):
    """GQA decode attention over the packed cache (R8, R9, R10).
    q_t: [B, Hq, 128] transformed queries.  Returns float64 [B, Hq, 128]."""
    q_t = np.asarray(q_t, dtype=np.float64)
    bsz, hq, d = q_t.shape
    g = hq // num_kv_heads
    out = np.zeros((bsz, hq, d))
    for b in range(bsz):
        n = int(ctx_len[b])
        if n <= 0:
            continue
        for kv in range(num_kv_heads):
            k_hat = dequant_groups(unpack_codes(cache["k_codes"][b, kv, :n], bits),
                                   cache["k_meta"][b, kv, :n], kind, bits)
            v_hat = dequant_groups(unpack_codes(cache["v_codes"][b, kv, :n], bits),
                                   cache["v_meta"][b, kv, :n], kind, bits)
            for h in range(kv * g, (kv + 1) * g):
                s = softmax_scale * (k_hat @ q_t[b, h])
                p = np.exp(s - np.max(s))
                p /= np.sum(p)
                out[b, h] = p @ v_hat
    return out


def decode_attention_pair(k_codes, k_meta, v_codes, v_meta, q_rows, softmax_scale, kind, bits):
    """Attention of the query rows [g, 128] of one (sequence, KV head) over n cached
    tokens (codes [n, 16b], meta [n, m]).  Same definition as decode_attention."""
    k_hat = dequant_groups(unpack_codes(k_codes, bits), k_meta, kind, bits)
    v_hat = dequant_groups(unpack_codes(v_codes, bits), v_meta, kind, bits)
    q_rows = np.asarray(q_rows, dtype=np.float64)
    out = np.zeros(q_rows.shape)
    if k_hat.shape[0] == 0:
        return out
    for i in range(q_rows.shape[0]):
        s = softmax_scale * (k_hat @ q_rows[i])
        p = np.exp(s - np.max(s))
        p /= np.sum(p)
        out[i] = p @ v_hat
    return out


def chunk_attention(cache, q_t, ctx_len, softmax_scale, kind, bits, num_kv_heads):
    """Causal attention of a chunk of n_q queries per sequence over the packed cache
    (R8, R9, R10, R18).  q_t: [B, n_q, Hq, 128] transformed queries; ctx_len counts the
    cached tokens including the chunk's own.  Returns float64 [B, n_q, Hq, 128]."""
    q_t = np.asarray(q_t, dtype=np.float64)
    bsz, nq, hq, d = q_t.shape
    g = hq // num_kv_heads
    capacity = cache["k_codes"].shape[2]
    out = np.zeros((bsz, nq, hq, d))
    for b in range(bsz):
        ctx = min(max(int(ctx_len[b]), 0), capacity)
        for kv in range(num_kv_heads):
            k_hat = dequant_groups(unpack_codes(cache["k_codes"][b, kv, :ctx], bits),
                                   cache["k_meta"][b, kv, :ctx], kind, bits)
            v_hat = dequant_groups(unpack_codes(cache["v_codes"][b, kv, :ctx], bits),
                                   cache["v_meta"][b, kv, :ctx], kind, bits)
            for i in range(nq):
                n = ctx - nq + i + 1          # positions 0 .. ctx - n_q + i
                if n <= 0:
                    continue
                for h in range(kv * g, (kv + 1) * g):
                    s = softmax_scale * (k_hat[:n] @ q_t[b, i, h])
                    p = np.exp(s - np.max(s))
                    p /= np.sum(p)
                    out[b, i, h] = p @ v_hat[:n]
    return out


# ------------------------------------------------------------------- paged layout
def gather_paged(pool, block_table, page_size):
    """Contiguous [B, Hkv, pages_per_seq * page_size, ...] copy of a paged pool
    [num_pages, Hkv, page_size, ...]: position t of sequence b is row t % page_size of
    page block_table[b, t // page_size].  (The paged layout is a serving-engine
    convention of this library, not a step of the method.)"""
    pool = np.asarray(pool)
    bt = np.asarray(block_table)
    b, pps = bt.shape
    out = np.empty((b, pool.shape[1], pps * page_size) + pool.shape[3:], dtype=pool.dtype)
    for s in range(b):
        for p in range(pps):
            out[s, :, p * page_size:(p + 1) * page_size] = pool[bt[s, p]]
    return out
