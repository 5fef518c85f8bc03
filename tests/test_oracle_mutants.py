"""Plant plausible mistakes in the CPU oracle and check that its pins catch each one.

Every mutant replaces one oracle function (module attribute, so the composite
functions pick it up) with a version carrying one typical slip: a transposed
operand, a wrong index or divisor, a wrong tie rule, a dropped term.  The test
passes when at least one pin fails on the mutant.
"""
import numpy as np
import pytest

import oracle.wushkv_oracle as orc
from tests import pins

_orig = {name: getattr(orc, name) for name in dir(orc) if callable(getattr(orc, name))}


def _transform_keys_transposed(k, tk):
    k = np.asarray(k, np.float64)
    x = np.empty_like(k)
    for h in range(tk.shape[0]):
        x[..., h, :] = k[..., h, :] @ np.asarray(tk[h], np.float64)      # T instead of T^T
    return x


def _transform_query_wrong_group(q, m, hkv):
    q = np.asarray(q, np.float64)
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        out[:, h, :] = q[:, h, :] @ np.asarray(m[h % hkv], np.float64).T   # h % Hkv
    return out


def _quest_pre_127(x, bits, alpha):
    x = np.asarray(x, np.float64)
    return alpha * np.sqrt(np.sum(x * x, -1) / 127) * 2.0 ** (1 - bits)


def _quest_pre_no_sqrt(x, bits, alpha):
    x = np.asarray(x, np.float64)
    return alpha * (np.sum(x * x, -1) / 128) * 2.0 ** (1 - bits)


def _quest_pre_wrong_exp(x, bits, alpha):
    x = np.asarray(x, np.float64)
    return alpha * np.sqrt(np.sum(x * x, -1) / 128) * 2.0 ** (-bits)


def _quest_codes_strict(x, delta, bits):
    x = np.asarray(x, np.float64)
    d = np.asarray(delta, np.float64)[..., None]
    half = 1 << (bits - 1)
    c = np.zeros(x.shape, np.uint8)
    for j in range(-(half - 1), half):
        c += (x > j * d).astype(np.uint8)                                  # > instead of >=
    return np.where(d == 0, np.uint8(half), c).astype(np.uint8)


def _quest_dequant_no_half(codes, delta, bits):
    return (np.asarray(codes, np.float64) - (1 << (bits - 1))) * np.asarray(delta)[..., None]


def _affine_pre_rank_off(x, bits, rlo, rhi):
    return _orig["affine_prerounding"](x, bits, rlo + 1, rhi - 1)


def _affine_pre_wrong_levels(x, bits, rlo, rhi):
    s, lo = _orig["affine_prerounding"](x, bits, rlo, rhi)
    return s * ((1 << bits) - 1) / (1 << bits), lo                        # / 2^b


def _affine_codes_half_up(x, scale, zero, bits):
    x = np.asarray(x, np.float64)
    s = np.asarray(scale, np.float64)[..., None]
    z = np.asarray(zero, np.float64)[..., None]
    c = np.zeros(x.shape, np.uint8)
    for j in range((1 << bits) - 1):
        c += (x >= z + (j + 0.5) * s).astype(np.uint8)                    # ties always up
    return np.where(s == 0, np.uint8(0), c).astype(np.uint8)


def _affine_dequant_no_zero(codes, scale, zero):
    return np.asarray(codes, np.float64) * np.asarray(scale)[..., None]


def _pack_msb(codes, bits):
    c = np.asarray(codes, np.uint8)
    planes = (c[..., :, None] >> np.arange(bits, dtype=np.uint8)) & 1
    flat = planes.reshape(c.shape[:-1] + (c.shape[-1] * bits,))
    return np.packbits(flat, axis=-1, bitorder="big")


def _unpack_msb(p, bits):
    p = np.asarray(p, np.uint8)
    flat = np.unpackbits(p, axis=-1, bitorder="big")
    planes = flat.reshape(p.shape[:-1] + (p.shape[-1] * 8 // bits, bits)).astype(np.uint8)
    return np.sum(planes << np.arange(bits, dtype=np.uint8), -1).astype(np.uint8)


def _fp16_truncate(x):
    x = np.asarray(x, np.float64)
    with np.errstate(over="ignore"):
        h = x.astype(np.float16).astype(np.float64)
    # one ulp toward zero where the library rounded away from zero
    lower = np.where(np.abs(h) > np.abs(x), np.nextafter(h.astype(np.float16), np.float16(0)).astype(np.float64), h)
    return lower


def _decode_scale_twice(cache, q_t, ctx, tau, kind, bits, hkv):
    return _orig["decode_attention"](cache, q_t, ctx, tau * tau * 11.3137, kind, bits, hkv)


def _decode_unnormalized(cache, q_t, ctx, tau, kind, bits, hkv):
    out = _orig["decode_attention"](cache, q_t, ctx, tau, kind, bits, hkv)
    return out * np.asarray([max(int(c), 1) for c in ctx])[:, None, None] ** 0.01


def _decode_wrong_group(cache, q_t, ctx, tau, kind, bits, hkv):
    q = np.asarray(q_t, np.float64)
    hq = q.shape[1]
    perm = [(h % hkv) * (hq // hkv) + h // hkv for h in range(hq)]        # interleaved groups
    return _orig["decode_attention"](cache, q[:, perm], ctx, tau, kind, bits, hkv)[:, np.argsort(perm)]


def _chunk_exclusive(cache, q_t, ctx, tau, kind, bits, hkv):
    """The query does not see its own position."""
    q = np.asarray(q_t, np.float64)
    nq = q.shape[1]
    return np.stack([orc.decode_attention(cache, q[:, i], [int(n) - nq + i for n in ctx], tau, kind, bits, hkv)
                     for i in range(nq)], axis=1)


def _chunk_not_causal(cache, q_t, ctx, tau, kind, bits, hkv):
    """Every query of the chunk sees the whole context."""
    q = np.asarray(q_t, np.float64)
    return np.stack([orc.decode_attention(cache, q[:, i], ctx, tau, kind, bits, hkv)
                     for i in range(q.shape[1])], axis=1)


def _chunk_positions_from_start(cache, q_t, ctx, tau, kind, bits, hkv):
    """Query i placed at position i instead of ctx - n_q + i."""
    q = np.asarray(q_t, np.float64)
    return np.stack([orc.decode_attention(cache, q[:, i], [min(i + 1, int(n)) for n in ctx], tau, kind, bits, hkv)
                     for i in range(q.shape[1])], axis=1)


def _rope_interleaved(k, cos, sin):
    """Pairs (2i, 2i + 1) instead of (i, i + 64)."""
    k = np.asarray(k, np.float64)
    ev, od = k[..., 0::2], k[..., 1::2]
    out = np.empty_like(k)
    out[..., 0::2] = ev * cos - od * sin
    out[..., 1::2] = od * cos + ev * sin
    return out


def _rope_wrong_sign(k, cos, sin):
    k = np.asarray(k, np.float64)
    lo, hi = k[..., :64], k[..., 64:]
    return np.concatenate([lo * cos + hi * sin, hi * cos - lo * sin], axis=-1)


def _append_rope_start_row(cache, k_pre, v_new, start_pos, tab, kind, bits, alpha=0.0, rlo=2, rhi=125, tk=None):
    """Every row of a sequence rotated with the table row of its first position."""
    k_pre = np.asarray(k_pre, np.float64)
    tab = np.asarray(tab, np.float64)
    k_rot = k_pre.copy()
    for b in range(k_pre.shape[0]):
        p = int(start_pos[b])
        k_rot[b] = orc.apply_rope(k_pre[b], tab[p, :64], tab[p, 64:])
    return orc.quantize_append(cache, k_rot, v_new, start_pos, kind, bits, alpha, rlo, rhi, tk=tk)


def _hadamard_transposed_blocks(n):
    """Sylvester recursion with the sign on the wrong block: [[H, -H], [H, H]]."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, -h], [h, h]])
    return h


def _hadamard_inv_t_unscaled(scale):
    """Inverse-transpose that forgets to invert the diagonal."""
    s = np.asarray(scale, np.float64)
    h = orc.hadamard(128) / np.sqrt(128)
    return np.stack([h * s[i][None, :] for i in range(s.shape[0])])


def _block_diag_transposed(blocks):
    """Each block placed transposed."""
    return _orig["block_diagonal_transform"](np.swapaxes(np.asarray(blocks), -1, -2))


def _pair_no_max_shift_wrong_scale(kc, km, vc, vm, q, tau, kind, bits):
    return _orig["decode_attention_pair"](kc, km, vc, vm, q, tau * 1.25, kind, bits)


def _gather_pages_by_modulo(pool, bt, ps):
    """Page index taken as t % pages_per_seq instead of t // page_size."""
    pool = np.asarray(pool)
    bt = np.asarray(bt)
    b, pps = bt.shape
    out = np.empty((b, pool.shape[1], pps * ps) + pool.shape[3:], dtype=pool.dtype)
    for s_ in range(b):
        for t in range(pps * ps):
            out[s_, :, t] = pool[bt[s_, t % pps], :, t % ps]
    return out


MUTANTS = {
    "transform_keys_transposed": {"transform_keys": _transform_keys_transposed},
    "transform_query_wrong_group": {"transform_query": _transform_query_wrong_group},
    "quest_rms_over_127": {"quest_step_prerounding": _quest_pre_127},
    "quest_no_sqrt": {"quest_step_prerounding": _quest_pre_no_sqrt},
    "quest_wrong_exponent": {"quest_step_prerounding": _quest_pre_wrong_exp},
    "quest_strict_compare": {"quest_codes": _quest_codes_strict},
    "quest_dequant_no_half": {"quest_dequant": _quest_dequant_no_half},
    "affine_rank_off_by_one": {"affine_prerounding": _affine_pre_rank_off},
    "affine_wrong_levels": {"affine_prerounding": _affine_pre_wrong_levels},
    "affine_ties_up": {"affine_codes": _affine_codes_half_up},
    "affine_dequant_no_zero": {"affine_dequant": _affine_dequant_no_zero},
    "pack_msb_first": {"pack_codes": _pack_msb, "unpack_codes": _unpack_msb},
    "fp16_truncate": {"fp16_round": _fp16_truncate},
    "decode_scale_wrong": {"decode_attention": _decode_scale_twice},
    "decode_unnormalized": {"decode_attention": _decode_unnormalized},
    "decode_wrong_group": {"decode_attention": _decode_wrong_group},
    "chunk_exclusive_window": {"chunk_attention": _chunk_exclusive},
    "chunk_not_causal": {"chunk_attention": _chunk_not_causal},
    "chunk_positions_from_start": {"chunk_attention": _chunk_positions_from_start},
    "rope_interleaved_pairs": {"apply_rope": _rope_interleaved},
    "rope_wrong_sign": {"apply_rope": _rope_wrong_sign},
    "append_rope_start_row": {"quantize_append_rope": _append_rope_start_row},
    "hadamard_wrong_sign_block": {"hadamard": _hadamard_transposed_blocks},
    "hadamard_inverse_unscaled": {"hadamard_diag_inverse_transpose": _hadamard_inv_t_unscaled},
    "block_diagonal_transposed": {"block_diagonal_transform": _block_diag_transposed},
    "decode_pair_scale_wrong": {"decode_attention_pair": _pair_no_max_shift_wrong_scale},
    "gather_page_index_modulo": {"gather_paged": _gather_pages_by_modulo},
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    for attr, fn in MUTANTS[name].items():
        monkeypatch.setattr(orc, attr, fn)
    failures = []
    for check in pins.ALL_PINS:
        try:
            check(orc)
        except AssertionError:
            failures.append(check.__name__)
        except Exception as e:  # a crash on the mutant also counts as caught
            failures.append(f"{check.__name__}:{type(e).__name__}")
    assert failures, f"mutant {name} passed every pin"
