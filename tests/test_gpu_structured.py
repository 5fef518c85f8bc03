"""GPU parity of wushkv_quantize_append_structured (block-diagonal and Hadamard-diagonal
key transforms, on decode-step appends and on larger ones through the tensor cores)
against the oracle's append with the same transform built as a dense T_k, and of
wushkv_transform_query_structured against the oracle's map by the dense inverse-transpose.

Bar, as for the other end-to-end appends: value codes and meta bit-exact; key meta may
differ by one fp16 ulp only within 1e-4 * Delta of an fp16 midpoint; key codes by +-1
only within 1e-4 * Delta of a decision threshold.  The block-diagonal kernel also gives
exactly what the dense decode-step kernel gives for the expanded matrix.
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


def _alpha(kind, bits):
    return QUEST_ALPHA[bits] if kind == orc.QUEST_INT else 0.0


def _blocks(hkv, bs, seed):
    """Well-conditioned blocks: orthogonal times a log-uniform diagonal scale."""
    rng = np.random.default_rng(seed)
    out = np.empty((hkv, 128 // bs, bs, bs))
    for h in range(hkv):
        for j in range(128 // bs):
            q, _ = np.linalg.qr(rng.standard_normal((bs, bs)))
            out[h, j] = q * np.exp(rng.uniform(np.log(0.25), np.log(4.0), bs))[None, :]
    return out.astype(np.float32)


def _scales(hkv, seed):
    rng = np.random.default_rng(seed)
    s = np.exp(rng.uniform(np.log(0.25), np.log(4.0), (hkv, 128))) * rng.choice([-1.0, 1.0], (hkv, 128))
    return s.astype(np.float32)


def _check(kind, bits, bsz, n, tkind, data, dense):
    w = QWEN8B_DECODE
    hkv = data.shape[0]
    start = [(7 * b) % 40 for b in range(bsz)]
    cap = max(64, max(start) + n)
    k = gen.keys(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    v = gen.values(w, 0, bsz, start, n)[:, :, :hkv].contiguous()
    alpha = _alpha(kind, bits)
    oc = orc.empty_cache(bsz, hkv, cap, kind, bits)
    assert orc.quantize_append(oc, gu.to_numpy64(k), gu.to_numpy64(v), start, kind, bits, alpha, 2, 125,
                               tk=dense) == 0
    cache = dq.PackedCache(bsz, hkv, cap, kind, bits, alpha)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    block = data.shape[-1] if tkind == dq.TRANSFORM_BLOCK_DIAG else 0
    dq.quantize_append_structured(cache, k.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32, device="cuda"),
                                  tkind, torch.from_numpy(data).cuda(), block=block, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gc = gu.cache_to_numpy(cache)
    np.testing.assert_array_equal(oc["v_codes"], gc["v_codes"])
    np.testing.assert_array_equal(oc["v_meta"], gc["v_meta"])
    x = orc.transform_keys(gu.to_numpy64(k), dense)
    flips, diffs, near = gu.check_key_rows(oc, gc, x, kind, bits, start, alpha)
    print(f"tkind={tkind} block={block} kind={kind} bits={bits} B={bsz} n={n}: meta flips {flips}, "
          f"code diffs {diffs} (near a boundary: {near})")
    return cache, k, v, start


@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("kind,bits", [(0, 2), (1, 2), (0, 4)])
@pytest.mark.parametrize("bsz,n", [(16, 1), (4, 16)])
def test_block_diagonal_append(bs, kind, bits, bsz, n):
    blocks = _blocks(2, bs, seed=bs + bits)
    dense = orc.block_diagonal_transform(blocks.astype(np.float64))
    _check(kind, bits, bsz, n, dq.TRANSFORM_BLOCK_DIAG, blocks, dense)


@pytest.mark.parametrize("kind,bits", [(0, 2), (0, 3), (1, 2), (1, 4)])
@pytest.mark.parametrize("bsz,n", [(16, 1), (4, 16)])
def test_hadamard_diagonal_append(kind, bits, bsz, n):
    s = _scales(2, seed=bits + 10 * kind)
    dense = orc.hadamard_diag_transform(s.astype(np.float64))
    _check(kind, bits, bsz, n, dq.TRANSFORM_HADAMARD_DIAG, s, dense)


def test_block_diagonal_equals_dense_decode_step_path():
    """Same four FMA chains over the block's terms: bit-identical to the dense kernel
    given the expanded matrix (whose other terms are exact zeros)."""
    blocks = _blocks(2, 32, seed=3)
    dense = orc.block_diagonal_transform(blocks.astype(np.float64)).astype(np.float32)
    cache, k, v, start = _check(1, 2, 16, 1, dq.TRANSFORM_BLOCK_DIAG, blocks, dense.astype(np.float64))
    ref = dq.PackedCache(16, 2, 64, 1, 2)
    dq.quantize_append(ref, k.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(dense).cuda())
    for a, b in zip(cache.tensors().values(), ref.tensors().values()):
        assert torch.equal(a, b)


@pytest.mark.parametrize("tkind,bs", [(2, 16), (2, 32), (2, 64), (3, 0)])
@pytest.mark.parametrize("kind,bits", [(0, 2), (1, 2), (0, 4)])
def test_structured_bulk_append(tkind, bs, kind, bits):
    """Appends of more than 64 rows (4 sequences x 64 tokens) take the tensor-core kernel
    with the structured transform expanded into its exact bf16 parts."""
    if tkind == dq.TRANSFORM_BLOCK_DIAG:
        data = _blocks(2, bs, seed=40 + bs + bits)
        dense = orc.block_diagonal_transform(data.astype(np.float64))
    else:
        data = _scales(2, seed=50 + bits + 10 * kind)
        dense = orc.hadamard_diag_transform(data.astype(np.float64))
    _check(kind, bits, 4, 64, tkind, data, dense)


def test_bulk_block_diagonal_equals_dense_bulk_path():
    """The expanded block-diagonal parts are the parts of the expanded dense matrix, so the
    tensor-core append gives identical bytes for both."""
    blocks = _blocks(2, 16, seed=8)
    dense = orc.block_diagonal_transform(blocks.astype(np.float64)).astype(np.float32)
    cache, k, v, start = _check(0, 2, 4, 64, dq.TRANSFORM_BLOCK_DIAG, blocks, dense.astype(np.float64))
    ref = dq.PackedCache(4, 2, cache.capacity, 0, 2, QUEST_ALPHA[2])
    dq.quantize_append(ref, k.cuda(), v.cuda(), torch.tensor(start, dtype=torch.int32, device="cuda"),
                       torch.from_numpy(dense).cuda())
    for a, b in zip(cache.tensors().values(), ref.tensors().values()):
        assert torch.equal(a, b)


@pytest.mark.parametrize("tkind,bs", [(2, 16), (2, 32), (2, 64), (3, 0)])
@pytest.mark.parametrize("qdtype", [torch.bfloat16, torch.float32])
def test_structured_query_map(tkind, bs, qdtype):
    """q' = T_k^{-T} q for the structured transforms against the oracle's map by the
    expanded dense inverse-transpose (fp32 arithmetic over <= 128 terms: 1e-5 relative)."""
    w = QWEN8B_DECODE
    hkv = w.num_kv_heads
    q = gen.queries(w).to(qdtype)
    if tkind == dq.TRANSFORM_BLOCK_DIAG:
        blocks = _blocks(hkv, bs, seed=60 + bs).astype(np.float64)
        inv_t = np.linalg.inv(blocks).transpose(0, 1, 3, 2)            # each block inverted, transposed
        data = np.ascontiguousarray(inv_t, dtype=np.float32)
        m = orc.block_diagonal_transform(data.astype(np.float64))
        # the dense inverse-transpose of the expanded key transform is the same matrix
        assert np.allclose(m, np.linalg.inv(orc.block_diagonal_transform(blocks)).transpose(0, 2, 1), atol=1e-5)
    else:
        data = _scales(hkv, seed=70)
        m = orc.hadamard_diag_inverse_transpose(data.astype(np.float64))
    got = dq.transform_query_structured(q.cuda(), tkind, torch.from_numpy(data).cuda(), hkv, block=bs)
    ref = orc.transform_query(gu.to_numpy64(q), m, hkv)
    err = np.abs(got.cpu().numpy() - ref) / (np.abs(ref).max(axis=-1, keepdims=True) + 1e-30)
    assert err.max() < 1e-5, err.max()
