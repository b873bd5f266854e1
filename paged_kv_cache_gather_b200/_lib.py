"""ctypes loader for ``libpagedkv.so`` and the C structs of ``include/pagedkv.h``.

The library is loaded on first use. If it is missing the call fails loudly:
there is no CPU or PyTorch fallback for any operation.
"""

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PAGEDKV_LIB", os.path.join(HERE, "libpagedkv.so"))

PKV_OK = 0
PKV_ERR_INVALID_ARG = -1
PKV_ERR_UNSUPPORTED = -2
PKV_ERR_CUDA = -3
PKV_ERR_WORKSPACE_TOO_SMALL = -4
PKV_ERR_BAD_INDEX = -5

PKV_DBG_BLOCK_ID = 1
PKV_DBG_SLOT = 2
PKV_DBG_LENGTH = 4
PKV_DBG_TIMEOUT = 8
PKV_DBG_QLEN_SUM = 16
PKV_DBG_OUT_OF_BLOCKS = 32
PKV_DBG_REFCOUNT = 64

PKV_F32 = 0
PKV_BF16 = 1
PKV_FP8_E4M3 = 2

PKV_MASK_NONE = 0
PKV_MASK_CAUSAL = 1
PKV_MASK_SLIDING = 2
PKV_MASK_PREFIX_LM = 3
PKV_MASK_DOCUMENT = 4

PKV_BLOCK_SKIP = 0
PKV_BLOCK_PARTIAL = 1
PKV_BLOCK_FULL = 2

# size of the fixed scratch of paged_attention_decode_noalloc (include/pagedkv.h)
PKV_NOALLOC_SCRATCH_BYTES = 8 << 20

# every symbol the header declares; the CPU test checks that all are exported
EXPORTS = (
    "paged_kv_append",
    "paged_kv_gather",
    "paged_kv_copy_blocks",
    "paged_kv_copy_blocks_fp8",
    "paged_attention_decode_workspace_size",
    "paged_attention_decode",
    "paged_attention_decode_append",
    "paged_attention_prefill",
    "paged_attention_decode_noalloc",
    "paged_attention_decode_shared_prefix_workspace_size",
    "paged_attention_decode_shared_prefix",
    "paged_attention_block_mask",
    "paged_kv_reserve_scratch_size",
    "paged_kv_reserve_slots",
    "paged_kv_reserve_slots_fp8",
    "paged_kv_append_fp8",
    "paged_attention_decode_fp8",
    "pkv_debug_wait_timeout",
    "pkv_status_string",
    "pkv_last_error",
    "pkv_version",
)


class MaskModC(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("window", ctypes.c_int32),
                ("window_per_seq", ctypes.c_void_p), ("window_per_head", ctypes.c_void_p),
                ("prefix_len", ctypes.c_void_p), ("doc_offsets", ctypes.c_void_p),
                ("doc_starts", ctypes.c_void_p)]


class CacheDescC(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class PagedKVError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(message)
        self.status = status


_lock = threading.Lock()
_lib = None

_i32 = ctypes.c_int32
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_f32 = ctypes.c_float


def _declare(lib):
    lib.paged_kv_append.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, CacheDescC, _vp, _vp]
    lib.paged_kv_append.restype = ctypes.c_int
    lib.paged_kv_gather.argtypes = [_vp, _vp, CacheDescC, _vp, _i32, _vp, _i32, _i32, _vp, _vp,
                                    _vp, _vp]
    lib.paged_kv_gather.restype = ctypes.c_int
    lib.paged_kv_copy_blocks.argtypes = [_vp, _vp, CacheDescC, _vp, _i32, _vp, _vp]
    lib.paged_kv_copy_blocks.restype = ctypes.c_int
    lib.paged_kv_copy_blocks_fp8.argtypes = [_vp, _vp, _vp, _vp, CacheDescC, _vp, _i32, _vp, _vp]
    lib.paged_kv_copy_blocks_fp8.restype = ctypes.c_int
    lib.paged_attention_decode_workspace_size.argtypes = [_i32, _i32, CacheDescC]
    lib.paged_attention_decode_workspace_size.restype = _sz
    lib.paged_attention_decode.argtypes = [_vp, _vp, _vp, CacheDescC, _vp, _i32, _vp, _i32, _i32,
                                           _f32, MaskModC, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.paged_attention_decode.restype = ctypes.c_int
    lib.paged_attention_decode_append.argtypes = [_vp, _vp, _vp, _vp, _vp, CacheDescC, _vp, _i32,
                                                  _vp, _i32, _i32, _f32, MaskModC, _vp, _vp, _vp,
                                                  _sz, _vp, _vp]
    lib.paged_attention_decode_append.restype = ctypes.c_int
    lib.paged_attention_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, CacheDescC, _vp, _i32, _vp,
                                            _vp, _i32, _i32, _i32, _f32, MaskModC, _vp, _vp, _vp,
                                            _vp]
    lib.paged_attention_prefill.restype = ctypes.c_int
    lib.paged_attention_decode_noalloc.argtypes = [_vp, _vp, _vp, CacheDescC, _vp, _i32, _vp, _i32,
                                                   _i32, _f32, MaskModC, _vp, _vp, _vp, _vp]
    lib.paged_attention_decode_noalloc.restype = ctypes.c_int
    lib.paged_attention_decode_shared_prefix_workspace_size.argtypes = [_i32, _i32, CacheDescC]
    lib.paged_attention_decode_shared_prefix_workspace_size.restype = _sz
    lib.paged_attention_decode_shared_prefix.argtypes = [
        _vp, _vp, _vp, CacheDescC, _vp, _i32, _vp, _i32, _i32, _f32, MaskModC, _vp, _i32, _i32,
        _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.paged_attention_decode_shared_prefix.restype = ctypes.c_int
    lib.paged_attention_block_mask.argtypes = [_vp, _vp, _i32, _i32, MaskModC, _i32, _i32, _i32,
                                               _i32, _vp, _vp]
    lib.paged_attention_block_mask.restype = ctypes.c_int
    lib.paged_kv_reserve_scratch_size.argtypes = [CacheDescC]
    lib.paged_kv_reserve_scratch_size.restype = _sz
    lib.paged_kv_reserve_slots.argtypes = [_vp, _vp, CacheDescC, _vp, _i32, _vp, _vp, _i32, _vp,
                                           _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp]
    lib.paged_kv_reserve_slots.restype = ctypes.c_int
    lib.paged_kv_reserve_slots_fp8.argtypes = [_vp, _vp, _vp, _vp, CacheDescC, _vp, _i32, _vp,
                                               _vp, _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                               _vp, _vp]
    lib.paged_kv_reserve_slots_fp8.restype = ctypes.c_int
    lib.paged_kv_append_fp8.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, CacheDescC, _vp,
                                        _vp]
    lib.paged_kv_append_fp8.restype = ctypes.c_int
    lib.paged_attention_decode_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, CacheDescC, _vp, _i32,
                                               _vp, _i32, _i32, _f32, MaskModC, _vp, _vp, _vp,
                                               _sz, _vp, _vp]
    lib.paged_attention_decode_fp8.restype = ctypes.c_int
    lib.pkv_debug_wait_timeout.argtypes = [_vp, _vp, _vp]
    lib.pkv_debug_wait_timeout.restype = ctypes.c_int
    lib.pkv_status_string.argtypes = [ctypes.c_int]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_last_error.argtypes = []
    lib.pkv_last_error.restype = ctypes.c_char_p
    lib.pkv_version.argtypes = []
    lib.pkv_version.restype = ctypes.c_int


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m paged_kv_cache_gather_b200.build` (no fallback exists)")
                handle = ctypes.CDLL(LIB_PATH)
                _declare(handle)
                _lib = handle
    return _lib


def check(status):
    if status != PKV_OK:
        l = lib()
        name = l.pkv_status_string(status).decode()
        msg = l.pkv_last_error().decode()
        raise PagedKVError(status, f"{name}: {msg}")
