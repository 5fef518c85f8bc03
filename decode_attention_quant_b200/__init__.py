"""WUSH-KV runtime hot path on B200: thin PyTorch-facing binding of libwushkv.so.

The functions below only check tensor shapes/dtypes and pass device pointers and
the current CUDA stream to the C ABI (include/wushkv.h); every step of the path
runs in the library's kernels.  PyTorch provides device memory and streams.

    cache = PackedCache(batch, num_kv_heads, capacity, kind=QUEST_INT, bits=2, clip_alpha=1.99)
    quantize_append(cache, k_new, v_new, start_pos, tk)          # keys post-RoPE
    q_t = transform_query(q, tk_inv_t, num_kv_heads)
    out = decode_attention(cache, q_t, ctx_len)
    out = chunk_attention(cache, q_t_chunk, ctx_len)              # [B, n_q, Hq, 128], causal
"""
import ctypes
import math

import torch

from . import _lib
from ._lib import (BF16, FP32, PCT_AFFINE, QUEST_INT, STATUS_BAD_PAGE, STATUS_CAPACITY,  # noqa: F401
                   STATUS_CTX_OVERFLOW, STATUS_META_OVERFLOW, STATUS_NONFINITE, STATUS_TIMEOUT,
                   TRANSFORM_BLOCK_DIAG, TRANSFORM_DENSE, TRANSFORM_HADAMARD_DIAG, WushkvError)

HEAD_DIM = 128

__all__ = ["PackedCache", "quantize_append", "quantize_append_rope", "quantize_append_structured", "transform_query",
           "transform_query_structured", "decode_attention",
           "decode_attention_noalloc", "decode_workspace_bytes", "chunk_attention", "chunk_workspace_bytes",
           "QUEST_INT", "PCT_AFFINE", "WushkvError", "library"]


def library():
    """The loaded ctypes library (raises ImportError if it was not built)."""
    return _lib.load()


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


class PackedCache:
    """Caller-owned packed KV cache of one layer (codes + fp16 meta), see wushkv_cache.

    Contiguous: tensors [batch, Hkv, capacity, ...].  Paged (page_size given): pools
    [num_pages, Hkv, page_size, ...] and an int32 block table [batch, capacity // page_size]
    whose row b lists the pages of sequence b in order."""

    def __init__(self, batch, num_kv_heads, capacity, kind=QUEST_INT, bits=2, clip_alpha=0.0,
                 rank_lo=2, rank_hi=125, device="cuda", tensors=None, page_size=None, num_pages=None,
                 block_table=None):
        self.batch, self.num_kv_heads, self.capacity = int(batch), int(num_kv_heads), int(capacity)
        self.kind, self.bits = int(kind), int(bits)
        self.clip_alpha, self.rank_lo, self.rank_hi = float(clip_alpha), int(rank_lo), int(rank_hi)
        self.page_size = None if page_size is None else int(page_size)
        self.block_table = None
        m = 1 if self.kind == QUEST_INT else 2
        if self.page_size is None:
            shp = (self.batch, self.num_kv_heads, self.capacity)
        else:
            if self.capacity % self.page_size:
                raise ValueError("capacity must be a multiple of page_size")
            self.pages_per_seq = self.capacity // self.page_size
            self.num_pages = int(num_pages if num_pages is not None else self.batch * self.pages_per_seq)
            if block_table is None:     # sequence b owns pages b * pages_per_seq ... in order
                block_table = torch.arange(self.batch * self.pages_per_seq, dtype=torch.int32).view(
                    self.batch, self.pages_per_seq)
            if tuple(block_table.shape) != (self.batch, self.pages_per_seq) or block_table.dtype != torch.int32:
                raise ValueError("block_table must be int32 [batch, capacity // page_size]")
            self.block_table = block_table.to(device if tensors is None else tensors["k_codes"].device).contiguous()
            shp = (self.num_pages, self.num_kv_heads, self.page_size)
        if tensors is None:
            self.k_codes = torch.zeros(shp + (16 * self.bits,), dtype=torch.uint8, device=device)
            self.v_codes = torch.zeros_like(self.k_codes)
            self.k_meta = torch.zeros(shp + (m,), dtype=torch.int16, device=device)
            self.v_meta = torch.zeros_like(self.k_meta)
        else:
            self.k_codes, self.v_codes = tensors["k_codes"], tensors["v_codes"]
            self.k_meta, self.v_meta = tensors["k_meta"], tensors["v_meta"]
            for name, t, last, dt in (("k_codes", self.k_codes, 16 * self.bits, torch.uint8),
                                      ("v_codes", self.v_codes, 16 * self.bits, torch.uint8),
                                      ("k_meta", self.k_meta, m, torch.int16),
                                      ("v_meta", self.v_meta, m, torch.int16)):
                if tuple(t.shape) != shp + (last,) or t.dtype != dt or not t.is_contiguous():
                    raise ValueError(f"{name}: expected contiguous {dt} {shp + (last,)}, got {t.dtype} {tuple(t.shape)}")

    @property
    def device(self):
        return self.k_codes.device

    def desc(self) -> _lib.CacheDesc:
        qp = _lib.QuantParams(self.kind, self.bits, self.clip_alpha, self.rank_lo, self.rank_hi)
        if self.page_size is None:
            paging = (None, 0, 0, 0)
        else:
            paging = (self.block_table.data_ptr(), self.pages_per_seq, self.page_size, self.num_pages)
        return _lib.CacheDesc(self.k_codes.data_ptr(), self.v_codes.data_ptr(), self.k_meta.data_ptr(),
                              self.v_meta.data_ptr(), self.batch, self.num_kv_heads, self.capacity,
                              HEAD_DIM, qp, *paging)

    def tensors(self):
        return {"k_codes": self.k_codes, "v_codes": self.v_codes, "k_meta": self.k_meta, "v_meta": self.v_meta}


def quantize_append(cache: PackedCache, k_new, v_new, start_pos, tk=None, status=None, stream=None):
    """Transform keys by tk (None = identity), quantize and pack K and V, write them at
    start_pos[b] + t.  k_new, v_new: [B, n_new, Hkv, 128] bf16 or fp32 on the cache's device."""
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    if k_new.dim() != 4 or k_new.shape[0] != cache.batch or k_new.shape[2] != cache.num_kv_heads \
            or k_new.shape[3] != HEAD_DIM:
        raise ValueError(f"k_new must be [B={cache.batch}, n, Hkv={cache.num_kv_heads}, 128]")
    if not (k_new.is_contiguous() and v_new.is_contiguous()):
        raise ValueError("k_new and v_new must be contiguous")
    if start_pos.dtype != torch.int32 or start_pos.numel() != cache.batch:
        raise ValueError("start_pos must be int32 [B]")
    if tk is not None and (tk.dtype != torch.float32 or tuple(tk.shape) != (cache.num_kv_heads, HEAD_DIM, HEAD_DIM)
                           or not tk.is_contiguous()):
        raise ValueError("tk must be contiguous float32 [Hkv, 128, 128]")
    d = cache.desc()
    rc = library().wushkv_quantize_append(ctypes.byref(d), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
                                          int(k_new.shape[1]), _ptr(start_pos), _ptr(tk), _ptr(status),
                                          _stream(cache.device, stream))
    _lib.check(rc, "wushkv_quantize_append")


def quantize_append_rope(cache: PackedCache, k_new, v_new, start_pos, rope_table, tk=None, status=None,
                         stream=None):
    """quantize_append with RoPE fused in front of the key transform: k_new holds pre-RoPE
    keys; the key of position p is rotated with rope_table[p] (fp32 [rows >= capacity, 128]:
    cos of the 64 pairs, then sin).  Decode-step appends only (bf16, B * n_new <= 64)."""
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    if k_new.dim() != 4 or k_new.shape[0] != cache.batch or k_new.shape[2] != cache.num_kv_heads \
            or k_new.shape[3] != HEAD_DIM:
        raise ValueError(f"k_new must be [B={cache.batch}, n, Hkv={cache.num_kv_heads}, 128]")
    if not (k_new.is_contiguous() and v_new.is_contiguous()):
        raise ValueError("k_new and v_new must be contiguous")
    if start_pos.dtype != torch.int32 or start_pos.numel() != cache.batch:
        raise ValueError("start_pos must be int32 [B]")
    if tk is not None and (tk.dtype != torch.float32 or tuple(tk.shape) != (cache.num_kv_heads, HEAD_DIM, HEAD_DIM)
                           or not tk.is_contiguous()):
        raise ValueError("tk must be contiguous float32 [Hkv, 128, 128]")
    if rope_table.dtype != torch.float32 or rope_table.dim() != 2 or rope_table.shape[1] != HEAD_DIM \
            or not rope_table.is_contiguous():
        raise ValueError("rope_table must be contiguous float32 [rows, 128]")
    d = cache.desc()
    rc = library().wushkv_quantize_append_rope(ctypes.byref(d), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
                                               int(k_new.shape[1]), _ptr(start_pos), _ptr(tk), _ptr(rope_table),
                                               int(rope_table.shape[0]), _ptr(status), _stream(cache.device, stream))
    _lib.check(rc, "wushkv_quantize_append_rope")


def quantize_append_structured(cache: PackedCache, k_new, v_new, start_pos, kind, data, block=0, status=None,
                               stream=None):
    """quantize_append with a structured key transform (kind = TRANSFORM_BLOCK_DIAG with
    data fp32 [Hkv, 128/block, block, block], or TRANSFORM_HADAMARD_DIAG with data = s fp32
    [Hkv, 128], T_k = H diag(s) / sqrt(128)); bf16 inputs (decode-step appends on the CUDA
    cores, larger ones on the tensor cores).  TRANSFORM_DENSE takes data as the dense T_k of
    quantize_append."""
    if k_new.shape != v_new.shape or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    if k_new.dim() != 4 or k_new.shape[0] != cache.batch or k_new.shape[2] != cache.num_kv_heads \
            or k_new.shape[3] != HEAD_DIM:
        raise ValueError(f"k_new must be [B={cache.batch}, n, Hkv={cache.num_kv_heads}, 128]")
    if not (k_new.is_contiguous() and v_new.is_contiguous()):
        raise ValueError("k_new and v_new must be contiguous")
    if start_pos.dtype != torch.int32 or start_pos.numel() != cache.batch:
        raise ValueError("start_pos must be int32 [B]")
    shapes = {_lib.TRANSFORM_DENSE: (cache.num_kv_heads, HEAD_DIM, HEAD_DIM),
              _lib.TRANSFORM_BLOCK_DIAG: (cache.num_kv_heads, HEAD_DIM // max(int(block), 1), int(block), int(block)),
              _lib.TRANSFORM_HADAMARD_DIAG: (cache.num_kv_heads, HEAD_DIM)}
    if int(kind) not in shapes:
        raise ValueError("unknown transform kind")
    if data.dtype != torch.float32 or tuple(data.shape) != shapes[int(kind)] or not data.is_contiguous():
        raise ValueError(f"transform data must be contiguous float32 {shapes[int(kind)]}")
    d = cache.desc()
    rc = library().wushkv_quantize_append_structured(ctypes.byref(d), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
                                                     int(k_new.shape[1]), _ptr(start_pos), int(kind), int(block),
                                                     _ptr(data), _ptr(status), _stream(cache.device, stream))
    _lib.check(rc, "wushkv_quantize_append_structured")


def transform_query(q, tk_inv_t, num_kv_heads, out=None, stream=None):
    """q' = T_k^{-T} q per query head (fp32 [B, Hq, 128])."""
    if q.dim() != 3 or q.shape[2] != HEAD_DIM or not q.is_contiguous():
        raise ValueError("q must be contiguous [B, Hq, 128]")
    if tk_inv_t.dtype != torch.float32 or tuple(tk_inv_t.shape) != (num_kv_heads, HEAD_DIM, HEAD_DIM) \
            or not tk_inv_t.is_contiguous():
        raise ValueError("tk_inv_t must be contiguous float32 [Hkv, 128, 128]")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    rc = library().wushkv_transform_query(_ptr(q), _dtype_code(q), q.shape[0], q.shape[1], int(num_kv_heads),
                                          _ptr(tk_inv_t), _ptr(out), _stream(q.device, stream))
    _lib.check(rc, "wushkv_transform_query")
    return out


def transform_query_structured(q, kind, data, num_kv_heads, block=0, out=None, stream=None):
    """q' = T_k^{-T} q for a structured key transform: kind = TRANSFORM_BLOCK_DIAG with data
    = the blocks of T_k^{-T} (fp32 [Hkv, 128/block, block, block]), TRANSFORM_HADAMARD_DIAG
    with data = the key transform's scales s (fp32 [Hkv, 128]), or TRANSFORM_DENSE with
    data = T_k^{-T} (fp32 [Hkv, 128, 128])."""
    if q.dim() != 3 or q.shape[2] != HEAD_DIM or not q.is_contiguous():
        raise ValueError("q must be contiguous [B, Hq, 128]")
    shapes = {_lib.TRANSFORM_DENSE: (num_kv_heads, HEAD_DIM, HEAD_DIM),
              _lib.TRANSFORM_BLOCK_DIAG: (num_kv_heads, HEAD_DIM // max(int(block), 1), int(block), int(block)),
              _lib.TRANSFORM_HADAMARD_DIAG: (num_kv_heads, HEAD_DIM)}
    if int(kind) not in shapes:
        raise ValueError("unknown transform kind")
    if data.dtype != torch.float32 or tuple(data.shape) != shapes[int(kind)] or not data.is_contiguous():
        raise ValueError(f"transform data must be contiguous float32 {shapes[int(kind)]}")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    rc = library().wushkv_transform_query_structured(_ptr(q), _dtype_code(q), q.shape[0], q.shape[1],
                                                     int(num_kv_heads), int(kind), int(block), _ptr(data),
                                                     _ptr(out), _stream(q.device, stream))
    _lib.check(rc, "wushkv_transform_query_structured")
    return out


def decode_workspace_bytes(cache: PackedCache, num_q_heads, num_splits=0) -> int:
    d = cache.desc()
    n = library().wushkv_decode_workspace_bytes(ctypes.byref(d), int(num_q_heads), int(num_splits))
    if n == 0:
        raise WushkvError(_lib.ERR_INVALID, "wushkv_decode_workspace_bytes")
    return int(n)


def decode_attention(cache: PackedCache, q_t, ctx_len, softmax_scale=None, out=None, workspace=None,
                     num_splits=0, status=None, stream=None):
    """Split-K GQA decode attention over the packed cache; fp32 [B, Hq, 128]."""
    if q_t.dtype != torch.float32 or q_t.dim() != 3 or q_t.shape[0] != cache.batch or q_t.shape[2] != HEAD_DIM \
            or not q_t.is_contiguous():
        raise ValueError("q_t must be contiguous float32 [B, Hq, 128]")
    if ctx_len.dtype != torch.int32 or ctx_len.numel() != cache.batch:
        raise ValueError("ctx_len must be int32 [B]")
    hq = int(q_t.shape[1])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(HEAD_DIM)
    if out is None:
        out = torch.empty(q_t.shape, dtype=torch.float32, device=q_t.device)
    need = decode_workspace_bytes(cache, hq, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q_t.device)
    d = cache.desc()
    rc = library().wushkv_decode_attention(ctypes.byref(d), _ptr(q_t), hq, _ptr(ctx_len), float(softmax_scale),
                                           _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           int(num_splits), _ptr(status), _stream(q_t.device, stream))
    _lib.check(rc, "wushkv_decode_attention")
    return out


def decode_attention_noalloc(cache: PackedCache, q_t, ctx_len, softmax_scale=None, out=None, num_splits=0,
                             status=None, stream=None):
    """decode_attention with the split partials in the library's fixed scratch array
    (no workspace is allocated; see wushkv_decode_attention_noalloc for the sharing rules)."""
    if q_t.dtype != torch.float32 or q_t.dim() != 3 or q_t.shape[0] != cache.batch or q_t.shape[2] != HEAD_DIM \
            or not q_t.is_contiguous():
        raise ValueError("q_t must be contiguous float32 [B, Hq, 128]")
    if ctx_len.dtype != torch.int32 or ctx_len.numel() != cache.batch:
        raise ValueError("ctx_len must be int32 [B]")
    hq = int(q_t.shape[1])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(HEAD_DIM)
    if out is None:
        out = torch.empty(q_t.shape, dtype=torch.float32, device=q_t.device)
    d = cache.desc()
    rc = library().wushkv_decode_attention_noalloc(ctypes.byref(d), _ptr(q_t), hq, _ptr(ctx_len),
                                                   float(softmax_scale), _ptr(out), int(num_splits),
                                                   _ptr(status), _stream(q_t.device, stream))
    if rc == _lib.ERR_WORKSPACE:
        raise WushkvError(rc, f"wushkv_decode_attention_noalloc: needs {decode_workspace_bytes(cache, hq, num_splits)} "
                              f"bytes of scratch, the fixed array holds {_lib.DECODE_STATIC_SCRATCH_BYTES}")
    _lib.check(rc, "wushkv_decode_attention_noalloc")
    return out


def chunk_workspace_bytes(cache: PackedCache, num_q_heads, n_q, num_splits=0) -> int:
    d = cache.desc()
    n = library().wushkv_chunk_workspace_bytes(ctypes.byref(d), int(num_q_heads), int(n_q), int(num_splits))
    if n == 0:
        raise WushkvError(_lib.ERR_INVALID, "wushkv_chunk_workspace_bytes")
    return int(n)


def chunk_attention(cache: PackedCache, q_t, ctx_len, softmax_scale=None, out=None, workspace=None,
                    num_splits=0, status=None, stream=None):
    """Causal attention of n_q chunk queries per sequence over the packed cache;
    q_t fp32 [B, n_q, Hq, 128] (query i at position ctx_len - n_q + i), returns the
    same shape."""
    if q_t.dtype != torch.float32 or q_t.dim() != 4 or q_t.shape[0] != cache.batch or q_t.shape[3] != HEAD_DIM \
            or not q_t.is_contiguous():
        raise ValueError("q_t must be contiguous float32 [B, n_q, Hq, 128]")
    if ctx_len.dtype != torch.int32 or ctx_len.numel() != cache.batch:
        raise ValueError("ctx_len must be int32 [B]")
    n_q, hq = int(q_t.shape[1]), int(q_t.shape[2])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(HEAD_DIM)
    if out is None:
        out = torch.empty(q_t.shape, dtype=torch.float32, device=q_t.device)
    if workspace is None:
        workspace = torch.empty(chunk_workspace_bytes(cache, hq, n_q, num_splits), dtype=torch.uint8,
                                device=q_t.device)
    d = cache.desc()
    rc = library().wushkv_chunk_attention(ctypes.byref(d), _ptr(q_t), n_q, hq, _ptr(ctx_len), float(softmax_scale),
                                          _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          int(num_splits), _ptr(status), _stream(q_t.device, stream))
    _lib.check(rc, "wushkv_chunk_attention")
    return out
