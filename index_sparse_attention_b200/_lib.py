"""ctypes binding of libsparse_attn.so (include/sparse_attn.h).

Argument marshalling only: the structs below mirror the C header field by field and
every step of the computation runs in the CUDA library.  Importing this module does
not need a GPU; calling into the library does.  A missing library is an error (there
is no fallback path).
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_attn.so")

SA_OK = 0
SA_ERR_INVALID = -1
SA_ERR_UNSUPPORTED = -2
SA_ERR_INDEX = -3
SA_ERR_ALIGN = -4
SA_ERR_CUDA = -5
SA_ERR_WORKSPACE = -7
SA_ERR_SCRATCH_LIMIT = -8
SA_ERR_DEVICE = -9
SA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
SA_TOPK_MAX_K = 4096

SA_MODE_DENSE, SA_MODE_BLOCK, SA_MODE_INDEX = 0, 1, 2
SA_FWD_FORM_AUTO, SA_FWD_FORM_ONE_HEAD, SA_FWD_FORM_CTA_PAIR, SA_FWD_FORM_TWO_HEADS = 0, 1, 2, 3
SA_FWD_FORM_TWO_TILES = 4
SA_BWD_FORM_AUTO, SA_BWD_FORM_SPLIT, SA_BWD_FORM_WHOLE = 0, 1, 2
SA_TILE = 128

STATUS_INDEX = 1
STATUS_TIMEOUT = 2
SA_STATUS_INDEX, SA_STATUS_TIMEOUT = STATUS_INDEX, STATUS_TIMEOUT

# every symbol include/sparse_attn.h declares
EXPORTS = (
    "index_to_block_sparse",
    "block_mask_to_block_sparse",
    "sparse_attn_fwd",
    "sparse_attn_fwd_gather",
    "sparse_attn_bwd_workspace_size",
    "sparse_attn_bwd",
    "sparse_attn_bwd_deterministic",
    "sparse_attn_bwd_noalloc",
    "sparse_attn_set_timing_events",
    "sparse_attn_set_wait_limit_ns",
    "sparse_attn_set_forward_form",
    "sparse_attn_set_backward_form",
    "sparse_attn_error_string",
    "topk_select",
)


class BlockSparseStruct(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32), ("causal", ctypes.c_int32), ("B", ctypes.c_int32),
        ("HK", ctypes.c_int32), ("Sq", ctypes.c_int64), ("Sk", ctypes.c_int64),
        ("bs", ctypes.c_int32), ("Mb", ctypes.c_int32), ("Nb", ctypes.c_int32),
        ("mask", ctypes.c_void_p), ("bitmap", ctypes.c_void_p), ("cnt", ctypes.c_void_p),
        ("idx", ctypes.c_void_p), ("tcnt", ctypes.c_void_p), ("tidx", ctypes.c_void_p),
    ]


class ParamsStruct(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("B", ctypes.c_int32), ("HQ", ctypes.c_int32), ("HK", ctypes.c_int32),
        ("Dqk", ctypes.c_int32), ("Dv", ctypes.c_int32), ("Sq", ctypes.c_int64),
        ("Sk", ctypes.c_int64), ("softmax_scale", ctypes.c_float),
        ("sparse", ctypes.POINTER(BlockSparseStruct)), ("dev_status", ctypes.c_void_p),
    ]


_lib = None


def load():
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m index_sparse_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, P_bs, P_p = ctypes.c_void_p, ctypes.POINTER(BlockSparseStruct), ctypes.POINTER(ParamsStruct)
    L.index_to_block_sparse.argtypes = [vp, ctypes.c_int32, P_bs, vp, vp]
    L.index_to_block_sparse.restype = ctypes.c_int
    L.block_mask_to_block_sparse.argtypes = [P_bs, vp]
    L.block_mask_to_block_sparse.restype = ctypes.c_int
    L.sparse_attn_fwd.argtypes = [P_p, vp]
    L.sparse_attn_fwd.restype = ctypes.c_int
    L.sparse_attn_fwd_gather.argtypes = [P_p, vp]
    L.sparse_attn_fwd_gather.restype = ctypes.c_int
    L.sparse_attn_bwd_workspace_size.argtypes = [P_p]
    L.sparse_attn_bwd_workspace_size.restype = ctypes.c_size_t
    L.sparse_attn_bwd.argtypes = [P_p, vp, ctypes.c_size_t, vp]
    L.sparse_attn_bwd.restype = ctypes.c_int
    L.sparse_attn_bwd_deterministic.argtypes = [P_p, vp, ctypes.c_size_t, vp]
    L.sparse_attn_bwd_deterministic.restype = ctypes.c_int
    L.sparse_attn_bwd_noalloc.argtypes = [P_p, vp]
    L.sparse_attn_bwd_noalloc.restype = ctypes.c_int
    L.sparse_attn_set_timing_events.argtypes = [vp]
    L.sparse_attn_set_timing_events.restype = ctypes.c_int
    L.sparse_attn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.sparse_attn_set_wait_limit_ns.restype = ctypes.c_int
    L.sparse_attn_set_forward_form.argtypes = [ctypes.c_int]
    L.sparse_attn_set_forward_form.restype = ctypes.c_int
    L.sparse_attn_set_backward_form.argtypes = [ctypes.c_int]
    L.sparse_attn_set_backward_form.restype = ctypes.c_int
    i64 = ctypes.c_int64
    L.topk_select.argtypes = [vp, i64, i64, i64, vp, vp, ctypes.c_int32, vp, vp, vp, vp]
    L.topk_select.restype = ctypes.c_int
    L.sparse_attn_error_string.argtypes = [ctypes.c_int]
    L.sparse_attn_error_string.restype = ctypes.c_char_p
    _lib = L
    return L


def error_string(code: int) -> str:
    return load().sparse_attn_error_string(code).decode()


class SparseAttnError(RuntimeError):
    def __init__(self, what, code):
        super().__init__(f"{what} failed: {error_string(code)} (code {code})")
        self.code = code


def check(what, code):
    if code != SA_OK:
        raise SparseAttnError(what, code)
