"""ctypes binding of libwushkv.so (the C ABI declared in include/wushkv.h).

Argument marshalling only.  The shared library is loaded from this package
directory; if it is missing the import fails loudly (there is no other
implementation to fall back to).
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwushkv.so")

OK = 0
ERR_INVALID = -1
ERR_UNSUPPORTED = -2
ERR_MISALIGNED = -3
ERR_WORKSPACE = -4
ERR_CUDA = -5

# size of the library's fixed decode scratch array (WUSHKV_DECODE_STATIC_SCRATCH_BYTES)
DECODE_STATIC_SCRATCH_BYTES = 8 << 20

QUEST_INT = 0
PCT_AFFINE = 1
BF16 = 0
FP32 = 1

STATUS_CAPACITY = 1
STATUS_NONFINITE = 2
STATUS_META_OVERFLOW = 4
STATUS_CTX_OVERFLOW = 8
STATUS_TIMEOUT = 16
STATUS_BAD_PAGE = 32
MAX_CHUNK = 16          # WUSHKV_MAX_CHUNK
TRANSFORM_DENSE, TRANSFORM_BLOCK_DIAG, TRANSFORM_HADAMARD_DIAG = 1, 2, 3   # wushkv_transform_kind

# every symbol include/wushkv.h declares
EXPORTS = (
    "wushkv_quantize_append",
    "wushkv_quantize_append_rope",
    "wushkv_quantize_append_structured",
    "wushkv_transform_query",
    "wushkv_transform_query_structured",
    "wushkv_decode_workspace_bytes",
    "wushkv_decode_attention",
    "wushkv_decode_attention_noalloc",
    "wushkv_chunk_workspace_bytes",
    "wushkv_chunk_attention",
    "wushkv_strerror",
    "wushkv_version",
)


class QuantParams(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("bits", ctypes.c_int32), ("clip_alpha", ctypes.c_double),
                ("rank_lo", ctypes.c_int32), ("rank_hi", ctypes.c_int32)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_meta", ctypes.c_void_p), ("v_meta", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("qp", QuantParams),
                ("block_table", ctypes.c_void_p), ("pages_per_seq", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class WushkvError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libwushkv.so not built ({path}); run python -m decode_attention_quant_b200.build")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cp = ctypes.POINTER(CacheDesc)
    lib.wushkv_quantize_append.argtypes = [cp, vp, vp, i32, i32, vp, vp, vp, vp]
    lib.wushkv_quantize_append.restype = ctypes.c_int
    lib.wushkv_quantize_append_rope.argtypes = [cp, vp, vp, i32, i32, vp, vp, vp, i32, vp, vp]
    lib.wushkv_quantize_append_rope.restype = ctypes.c_int
    lib.wushkv_quantize_append_structured.argtypes = [cp, vp, vp, i32, i32, vp, i32, i32, vp, vp, vp]
    lib.wushkv_quantize_append_structured.restype = ctypes.c_int
    lib.wushkv_transform_query.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
    lib.wushkv_transform_query.restype = ctypes.c_int
    lib.wushkv_transform_query_structured.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    lib.wushkv_transform_query_structured.restype = ctypes.c_int
    lib.wushkv_decode_workspace_bytes.argtypes = [cp, i32, i32]
    lib.wushkv_decode_workspace_bytes.restype = sz
    lib.wushkv_decode_attention.argtypes = [cp, vp, i32, vp, ctypes.c_float, vp, vp, sz, i32, vp, vp]
    lib.wushkv_decode_attention.restype = ctypes.c_int
    lib.wushkv_decode_attention_noalloc.argtypes = [cp, vp, i32, vp, ctypes.c_float, vp, i32, vp, vp]
    lib.wushkv_decode_attention_noalloc.restype = ctypes.c_int
    lib.wushkv_chunk_workspace_bytes.argtypes = [cp, i32, i32, i32]
    lib.wushkv_chunk_workspace_bytes.restype = sz
    lib.wushkv_chunk_attention.argtypes = [cp, vp, i32, i32, vp, ctypes.c_float, vp, vp, sz, i32, vp, vp]
    lib.wushkv_chunk_attention.restype = ctypes.c_int
    lib.wushkv_strerror.argtypes = [ctypes.c_int]
    lib.wushkv_strerror.restype = ctypes.c_char_p
    lib.wushkv_version.argtypes = []
    lib.wushkv_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().wushkv_strerror(int(code)).decode()


def check(code: int, where: str):
    if code != OK:
        raise WushkvError(code, where)
