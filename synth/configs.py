"""Workload descriptions for the WUSH-KV runtime hot path (shapes and quantizer settings).

Plain data only: shapes, bit widths, clip multipliers and percentile ranks.  No step
of the method is computed here.  The five workloads mirror the ones the WUSH-KV
summary pages motivate: a tiny single-layer case, a Qwen3-8B-shaped decode layer
(32 query / 8 KV heads, head_dim 128), a QuEST bit-width sweep, a 131k-token
long-context decode, and a 64-layer Qwen3-32B-shaped stack (64 query / 8 KV heads).
The quantizers are the two the pages name (ai4snews page, paragraphs 3-4): a
QuEST-INT-style RMS-clipped symmetric grid and an OSCAR-style percentile-clipped
affine grid, both per (token, head) group of 128 values.
"""
from dataclasses import dataclass, field
from typing import Tuple

QUEST_INT = 0
PCT_AFFINE = 1

HEAD_DIM = 128
# clip multipliers of the QuEST-INT-style grid for 2, 3 and 4 bits
QUEST_ALPHA = {2: 1.99, 3: 2.34, 4: 2.68}
# 0-based ascending ranks of the percentile-clipped affine grid (128-value groups)
AFFINE_RANKS = (2, 125)


@dataclass(frozen=True)
class QuantSpec:
    kind: int
    bits: int
    clip_alpha: float = 0.0
    rank_lo: int = AFFINE_RANKS[0]
    rank_hi: int = AFFINE_RANKS[1]

    @property
    def meta_per_group(self) -> int:
        return 1 if self.kind == QUEST_INT else 2

    @property
    def code_bytes(self) -> int:
        return 16 * self.bits


def quest(bits: int) -> QuantSpec:
    return QuantSpec(QUEST_INT, bits, QUEST_ALPHA[bits])


def affine(bits: int = 2) -> QuantSpec:
    return QuantSpec(PCT_AFFINE, bits, 0.0, *AFFINE_RANKS)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    ctx: int                 # context length seen by the decode step
    quant: QuantSpec
    layers: int = 1
    history: int = 0         # tokens appended (untimed) before the timed append
    append_tokens: int = 0   # tokens per sequence in the timed append
    key_outliers: Tuple[int, ...] = (3, 17, 64, 100)
    key_outlier_gain: float = 20.0
    value_heavy: Tuple[int, ...] = ()
    value_heavy_gain: float = 10.0
    rope_theta: float = 1.0e6
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


# Tiny single layer; history = the 256 prompt tokens, QuEST 2-bit
TINY = Workload("tiny_b1_h4kv1_t256_quest2", batch=1, num_q_heads=4, num_kv_heads=1,
                ctx=256, quant=quest(2), history=0, append_tokens=256, seed=1000)
# Qwen3-8B-shaped decode layer, percentile-affine 2-bit
QWEN8B_DECODE = Workload("qwen3_8b_b16_ctx32768_affine2", batch=16, num_q_heads=32,
                         num_kv_heads=8, ctx=32768, quant=affine(2), history=32767,
                         append_tokens=1, value_heavy=(3, 17), seed=2000)
# QuEST bit-width sweep on the Qwen3-8B shapes: 2048-token chunk appended after 30720
def QWEN8B_SWEEP(bits: int) -> Workload:
    return Workload(f"qwen3_8b_b16_chunk2048_quest{bits}", batch=16, num_q_heads=32,
                    num_kv_heads=8, ctx=32768, quant=quest(bits), history=30720,
                    append_tokens=2048, value_heavy=(3, 17), seed=3000 + bits)
# Long-context decode, split-K
QWEN8B_LONG = Workload("qwen3_8b_b4_ctx131072_affine2", batch=4, num_q_heads=32,
                       num_kv_heads=8, ctx=131072, quant=affine(2), history=131071,
                       append_tokens=1, value_heavy=(3, 17), seed=4000)
# Qwen3-32B-shaped 64-layer stack, 16-token chunk per layer
QWEN32B_STACK = Workload("qwen3_32b_64l_b32_ctx8192_quest2", batch=32, num_q_heads=64,
                         num_kv_heads=8, ctx=8192, quant=quest(2), layers=64,
                         history=8176, append_tokens=16, value_heavy=(3, 17), seed=5000)

ALL = [TINY, QWEN8B_DECODE, QWEN8B_SWEEP(2), QWEN8B_SWEEP(3), QWEN8B_SWEEP(4),
       QWEN8B_LONG, QWEN32B_STACK]
