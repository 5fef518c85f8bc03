"""The 64-layer Qwen3-32B-shaped stack (batch 32, 64 query / 8 KV heads, context 8192,
QuEST 2-bit), end to end as the benchmark runs it: each layer has its own seed and T_k,
its cache holds 8176 tokens appended by the GPU, and one step runs, per layer, the
append of a 16-token chunk, the query map by T_k^{-T} and decode attention, all 64
layers captured in one CUDA graph and replayed.

Checked on layers 0, 31 and 63: the chunk's value codes and meta bit-exact against the
oracle's append of the same inputs, its key codes and meta under the end-to-end rule
(+-1 / one fp16 ulp only within 1e-4 * Delta of a boundary, counts printed), and the
decode output of every (sequence, KV head) pair against the oracle on the GPU's codes
(max-abs <= 2e-3, relative L2 <= 1e-2).
"""
import math

import numpy as np
import pytest
import torch

import decode_attention_quant_b200 as dq
import oracle.wushkv_oracle as orc
from synth import gen
from synth.configs import QWEN32B_STACK
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu
TAU = 1.0 / math.sqrt(128)
MAX_ABS, REL_L2 = 2e-3, 1e-2
CHECKED = (0, 31, 63)


def test_qwen32b_stack_64_layers_in_one_graph():
    w = QWEN32B_STACK
    qs = w.quant
    dev = torch.device("cuda")
    n = w.append_tokens
    start = torch.full((w.batch,), w.history, dtype=torch.int32, device=dev)
    ctx = torch.full((w.batch,), w.ctx, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    layers = []
    for layer in range(w.layers):
        tk, tinv = gen.transforms(w, layer)
        cache = dq.PackedCache(w.batch, w.num_kv_heads, w.ctx, qs.kind, qs.bits, qs.clip_alpha)
        tk_d = torch.from_numpy(tk).to(dev)
        assert gu.append_history(cache, w, w.history, tk_d, layer=layer) == 0
        k = gen.keys(w, 0, w.batch, w.history, n, layer=layer, device=dev, salt=1)
        v = gen.values(w, 0, w.batch, w.history, n, layer=layer, device=dev, salt=1)
        q = gen.queries(w, layer, device=dev).contiguous()
        q_t = torch.empty(q.shape, dtype=torch.float32, device=dev)
        out = torch.empty_like(q_t)
        ws = torch.empty(dq.decode_workspace_bytes(cache, w.num_q_heads), dtype=torch.uint8, device=dev)
        layers.append(dict(cache=cache, tk=tk, tk_d=tk_d, tinv_d=torch.from_numpy(tinv).to(dev), k=k, v=v, q=q,
                           q_t=q_t, out=out, ws=ws))

    def step():
        for L in layers:
            dq.quantize_append(L["cache"], L["k"], L["v"], start, L["tk_d"], status)
            dq.transform_query(L["q"], L["tinv_d"], w.num_kv_heads, out=L["q_t"])
            dq.decode_attention(L["cache"], L["q_t"], ctx, TAU, out=L["out"], workspace=L["ws"], status=status)

    step()                                   # warm-up (and the appends' first write)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for L in layers:
        L["out"].zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert status.item() == 0

    for layer in CHECKED:
        L = layers[layer]
        cn = gu.cache_to_numpy(L["cache"])
        # the chunk appended this step, against the oracle's append of the same inputs
        oc = orc.empty_cache(w.batch, w.num_kv_heads, n, qs.kind, qs.bits)
        k64, v64 = gu.to_numpy64(L["k"]), gu.to_numpy64(L["v"])
        assert orc.quantize_append(oc, k64, v64, [0] * w.batch, qs.kind, qs.bits, qs.clip_alpha,
                                   tk=L["tk"].astype(np.float64)) == 0
        rows = slice(w.history, w.history + n)
        gc = {name: a[:, :, rows] for name, a in cn.items()}
        for name in ("v_codes", "v_meta"):
            assert np.array_equal(oc[name], gc[name]), (layer, name)
        x = orc.transform_keys(k64, L["tk"].astype(np.float64))
        flips, diffs, near = gu.check_key_rows(oc, gc, x, qs.kind, qs.bits, [0] * w.batch, qs.clip_alpha)
        # decode of every pair on the GPU's codes, with the GPU's query map
        ma, rl, npairs = gu.decode_vs_oracle(cn, L["q_t"].cpu().numpy().astype(np.float64), ctx.cpu().numpy(), TAU,
                                             qs.kind, qs.bits, w.num_kv_heads, L["out"].cpu().numpy())
        print(f"layer {layer}: chunk key meta flips {flips}, key code diffs {diffs} (near a boundary {near}); "
              f"decode {npairs} pairs, worst max-abs {ma:.3e}, rel-L2 {rl:.3e}")
        assert npairs == w.batch * w.num_kv_heads
        assert ma <= MAX_ABS and rl <= REL_L2
    del graph
