"""Seeded synthetic inputs for the WUSH-KV runtime hot path.

This module only draws random numbers and lays them out; it computes no step of
the method (no key transform, no quantizer, no attention).  Both the CUDA path
and the CPU oracle consume the exact bytes it returns.

Recipe (the WUSH-KV pages print no data, so every input is synthetic):
  * key transform per (layer, KV head): T_k = Q1 diag(s) Q2 with Q1, Q2
    Haar-orthogonal (QR of a Gaussian matrix, signs of diag(R) folded into Q) and
    s log-uniform in [0.25, 4].  Its inverse-transpose is Q1 diag(1/s) Q2 (closed
    form, fp64).  Both are rounded once to fp32.  A general invertible T_k is what
    the ai4snews page (paragraph 1) says WUSH-KV allows, unlike orthogonal methods.
  * keys: N(0,1) per element times a per-(layer, KV head, channel) factor
    exp(N(0,1)), channels {3,17,64,100} times 20 more, then rotate-half RoPE with
    theta = 1e6 at each token's absolute position, in fp64, then rounded to bf16.
    The transform is applied after RoPE (ai4snews page, paragraph 4), so the keys
    handed to the hot path are post-RoPE.
  * values: bf16 N(0,1), optional heavy channels times 10.
  * queries: bf16 N(0,1), taken as already post-RoPE.
  * random caches (decode-only tests): uniform random code bytes and fp16 meta
    drawn from a stated range.
"""
import math
import numpy as np
import torch

from .configs import HEAD_DIM, QUEST_INT, Workload

_D = HEAD_DIM


def _np_rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def _torch_gen(device, *key) -> torch.Generator:
    seed = int(np.random.SeedSequence([int(k) for k in key]).generate_state(1, np.uint64)[0] >> 1)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def haar_orthogonal(rng: np.random.Generator, n: int = _D) -> np.ndarray:
    z = rng.standard_normal((n, n))
    q, r = np.linalg.qr(z)
    return q * np.sign(np.diag(r))[None, :]


def key_transform_pair(rng: np.random.Generator, n: int = _D):
    """Return (T_k, T_k^{-T}) in fp64 from one draw: Q1 diag(s) Q2 and Q1 diag(1/s) Q2."""
    q1 = haar_orthogonal(rng, n)
    q2 = haar_orthogonal(rng, n)
    s = np.exp(rng.uniform(math.log(0.25), math.log(4.0), size=n))
    t = (q1 * s[None, :]) @ q2
    t_inv_t = (q1 / s[None, :]) @ q2
    return t, t_inv_t


def transforms(w: Workload, layer: int = 0):
    """fp32 arrays [Hkv][128][128] (row-major) of T_k and T_k^{-T} for one layer."""
    tk = np.empty((w.num_kv_heads, _D, _D), np.float32)
    tinv = np.empty_like(tk)
    for h in range(w.num_kv_heads):
        t, ti = key_transform_pair(_np_rng(w.seed, layer, h, 11))
        tk[h] = t.astype(np.float32)
        tinv[h] = ti.astype(np.float32)
    return tk, tinv


def key_channel_scale(w: Workload, layer: int = 0) -> np.ndarray:
    """fp64 [Hkv][128]: exp(N(0,1)) per channel, outlier channels times the gain."""
    rng = _np_rng(w.seed, layer, 12)
    s = np.exp(rng.standard_normal((w.num_kv_heads, _D)))
    for c in w.key_outliers:
        s[:, c] *= w.key_outlier_gain
    return s


def rope_tables(positions: torch.Tensor, theta: float):
    """cos/sin fp64 [..., 64] of the rotate-half RoPE at the given positions."""
    i = torch.arange(_D // 2, dtype=torch.float64, device=positions.device)
    inv_freq = theta ** (-2.0 * i / _D)
    ang = positions.to(torch.float64)[..., None] * inv_freq
    return torch.cos(ang), torch.sin(ang)


def keys(w: Workload, b0: int, b1: int, t0, n: int, layer: int = 0, device="cpu",
         salt: int = 0, rope: bool = True) -> torch.Tensor:
    """Post-RoPE bf16 keys [b1-b0][n][Hkv][128] for positions t0..t0+n-1 (rope=False:
    the same draws before RoPE, rounded once to bf16).

    t0 is an int or a per-sequence int sequence of start positions.
    """
    g = _torch_gen(device, w.seed, layer, b0, b1, int(np.sum(t0)), n, salt, 13)
    nb = b1 - b0
    k = torch.randn((nb, n, w.num_kv_heads, _D), generator=g, device=device, dtype=torch.float64)
    k *= torch.as_tensor(key_channel_scale(w, layer), device=device)[None, None]
    if not rope:
        return k.to(torch.float32).to(torch.bfloat16)
    starts = torch.as_tensor(np.broadcast_to(np.asarray(t0, np.int64), (nb,)).copy(), device=device)
    pos = starts[:, None] + torch.arange(n, device=device)[None, :]
    cos, sin = rope_tables(pos, w.rope_theta)
    cos = cos[:, :, None, :]
    sin = sin[:, :, None, :]
    lo, hi = k[..., : _D // 2], k[..., _D // 2:]
    out = torch.cat([lo * cos - hi * sin, hi * cos + lo * sin], dim=-1)
    return out.to(torch.float32).to(torch.bfloat16)


def values(w: Workload, b0: int, b1: int, t0, n: int, layer: int = 0, device="cpu",
           salt: int = 0) -> torch.Tensor:
    """bf16 values [b1-b0][n][Hkv][128]: N(0,1), heavy channels times the gain."""
    g = _torch_gen(device, w.seed, layer, b0, b1, int(np.sum(t0)), n, salt, 14)
    v = torch.randn((b1 - b0, n, w.num_kv_heads, _D), generator=g, device=device,
                    dtype=torch.float32)
    for c in w.value_heavy:
        v[..., c] *= w.value_heavy_gain
    return v.to(torch.bfloat16)


def rope_table(rows: int, theta: float) -> torch.Tensor:
    """fp32 [rows][128] cos/sin cache of a serving engine: row p = cos of the 64
    rotate-half pairs at position p, then their sin (computed in fp64, rounded once)."""
    cos, sin = rope_tables(torch.arange(rows), theta)
    return torch.cat([cos, sin], dim=-1).to(torch.float32).contiguous()


def queries(w: Workload, layer: int = 0, device="cpu", salt: int = 0) -> torch.Tensor:
    """bf16 decode queries [B][Hq][128], N(0,1)."""
    g = _torch_gen(device, w.seed, layer, salt, 15)
    q = torch.randn((w.batch, w.num_q_heads, _D), generator=g, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16)


def fp32_groups(shape, seed: int, device="cpu", heavy_tail: bool = True) -> torch.Tensor:
    """fp32 pre-transformed group values (quantizer-only tests): N(0,1) times
    exp(N(0,1)) per group, with a few large outliers per group when heavy_tail."""
    g = _torch_gen(device, seed, 16)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    scale = torch.exp(torch.randn(shape[:-1] + (1,), generator=g, device=device))
    x = x * scale
    if heavy_tail:
        idx = torch.randint(0, shape[-1], shape[:-1] + (2,), generator=g, device=device)
        x.scatter_(-1, idx, x.gather(-1, idx) * 15.0)
    return x.contiguous()


def random_cache(batch: int, num_kv_heads: int, capacity: int, kind: int, bits: int,
                 seed: int, device="cpu", k_scale_range=(1.0, 3.0), v_scale_range=(0.5, 1.5)):
    """Random packed cache for decode-only tests.

    Codes: uniform random bytes.  Meta (fp16 bit patterns): QuEST step in the stated
    range; affine scale in the range and zero = -(2^b-1)/2 * scale * U(0.8, 1.2).
    Returns dict of uint8/int16 tensors: k_codes, v_codes [B][Hkv][T][16b],
    k_meta, v_meta [B][Hkv][T][m].
    """
    g = _torch_gen(device, seed, 17)
    m = 1 if kind == QUEST_INT else 2
    shp = (batch, num_kv_heads, capacity)
    out = {}
    for side, rng_ in (("k", k_scale_range), ("v", v_scale_range)):
        out[f"{side}_codes"] = torch.randint(0, 256, shp + (16 * bits,), generator=g,
                                             device=device, dtype=torch.uint8)
        lo, hi = rng_
        s = lo + (hi - lo) * torch.rand(shp, generator=g, device=device, dtype=torch.float32)
        if m == 1:
            meta = s[..., None]
        else:
            z = -((1 << bits) - 1) / 2.0 * s * (0.8 + 0.4 * torch.rand(shp, generator=g, device=device))
            meta = torch.stack([s, z], dim=-1)
        out[f"{side}_meta"] = meta.to(torch.float16).view(torch.int16).contiguous()
    return out
