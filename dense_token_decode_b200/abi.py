"""ctypes binding of libfs (include/fs.h): the same names, argument
marshalling only. Every step of the forward pass runs in libfs's kernels.

Loading fails loudly (``LibraryMissing``) when ``libfs.so`` has not been
built: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes as C
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfs.so")

FS_OK = 0
FS_ERR_INVALID = -1
FS_ERR_NULL = -2
FS_ERR_ALIGN = -3
FS_ERR_OOM = -4
FS_ERR_EMPTY = -5
FS_ERR_TOKEN = -6
FS_ERR_CONTEXT = -7
FS_ERR_CUDA = -8
FS_ERR_SEQ = -9
FS_ERR_DEVICE = -10
FS_ERR_UNSUPPORTED = -11

FS_WEIGHT_BF16 = 0
FS_WEIGHT_Q8_0 = 1

FS_STOP_EOS = 1
FS_STOP_BUDGET = 2
FS_STOP_CONTEXT = 3


class fs_config(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("ffn", C.c_int32),
                ("vocab", C.c_int32), ("rms_eps", C.c_float), ("rope_theta", C.c_double),
                ("max_pos", C.c_int32), ("weight_format", C.c_int32)]


class fs_linear(C.Structure):
    _fields_ = [("data", C.c_void_p), ("scales", C.c_void_p)]


class fs_layer_weights(C.Structure):
    _fields_ = [("wq", fs_linear), ("wk", fs_linear), ("wv", fs_linear), ("wo", fs_linear),
                ("wg", fs_linear), ("wu", fs_linear), ("wd", fs_linear),
                ("attn_norm", C.c_void_p), ("ffn_norm", C.c_void_p),
                ("q_norm", C.c_void_p), ("k_norm", C.c_void_p)]


class fs_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("final_norm", C.c_void_p),
                ("layers", C.POINTER(fs_layer_weights))]


class LibraryMissing(RuntimeError):
    pass


_P = C.c_void_p
_I = C.c_int32
_PI = C.POINTER(C.c_int32)

# name -> (restype, argtypes)
SIGNATURES = {
    "fs_model_create": (_I, [C.POINTER(fs_config), C.POINTER(fs_weights), C.POINTER(_P)]),
    "fs_model_destroy": (None, [_P]),
    "fs_kv_alloc": (_I, [_P, _I, _I, C.POINTER(_P)]),
    "fs_kv_free": (None, [_P]),
    "fs_kv_reset": (_I, [_P, _I]),
    "fs_kv_length": (_I, [_P, _I, _PI]),
    "fs_kv_import": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "fs_kv_export": (_I, [_P, _I, _I, _I, _I, _P, _P, _P]),
    "fs_kv_set_length": (_I, [_P, _I, _I]),
    "fs_prefill": (_I, [_P, _P, _I, _P, _I, _P, _P, _P]),
    "fs_decode_step": (_I, [_P, _P, _P, _P, _I, _P, _P, _P]),
    "fs_forward_batch": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P]),
    "fs_greedy": (_I, [_P, _P, _I, _P, _I, _I, _P, _I, _P, _PI, _PI, _P]),
    "fs_sample": (_I, [_P, _P, _I, C.c_float, _I, C.c_float, C.c_uint64, C.c_uint64, _P, _P]),
    "fs_generate": (_I, [_P, _P, _I, _P, _I, _I, _P, _I, C.c_float, _I, C.c_float, C.c_uint64,
                         _P, _PI, _PI, _P]),
    "fs_debug_capture": (_I, [_P, _P, _I]),
    "fs_debug_block": (_I, [_P, _P, _I, _I, _P, _I, _P, _P]),
    "fs_debug_dequant_q8_0": (_I, [_P, _P, _I, _I, _P, _P]),
    "fs_debug_trace": (_I, [_P, _P]),
    "fs_debug_wait_limit": (_I, [_P, C.c_uint64, _I]),
    "fs_debug_decode_path": (_I, [_P, _I]),
    "fs_debug_decode_kernel": (_I, [_P, _I, _PI]),
    "fs_debug_lm_head": (_I, [_P, _P, _I, _P, _P, _P]),
    "fs_device_error": (_I, [_P, _PI]),
    "fs_set_prefill_split": (_I, [_P, _I]),
    "fs_lm_head_argmax_noalloc": (_I, [_P, _P, _I, _I, C.c_float, _P, _I, _P, _P, _P]),
    "fs_debug_kernel_launches": (C.c_uint64, []),
    "fs_last_error_string": (C.c_char_p, []),
    "fs_status_string": (C.c_char_p, [_I]),
}

_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load() -> C.CDLL:
    """Load libfs.so (once). Raises LibraryMissing if it was never built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise LibraryMissing(f"{_LIB_PATH} is missing: run `python -m dense_token_decode_b200.build`")
    lib = C.CDLL(_LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class FsError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        name = lib.fs_status_string(status).decode()
        msg = lib.fs_last_error_string().decode()
        super().__init__(f"{where}: {name} ({status}): {msg}")
        self.status = status


def check(status: int, where: str) -> int:
    if status != FS_OK:
        raise FsError(status, where)
    return status


def _wrap(name):
    def call(*args):
        return getattr(load(), name)(*args)
    call.__name__ = name
    call.__doc__ = f"libfs {name} (see include/fs.h)."
    return call


fs_model_create = _wrap("fs_model_create")
fs_model_destroy = _wrap("fs_model_destroy")
fs_kv_alloc = _wrap("fs_kv_alloc")
fs_kv_free = _wrap("fs_kv_free")
fs_kv_reset = _wrap("fs_kv_reset")
fs_kv_length = _wrap("fs_kv_length")
fs_kv_import = _wrap("fs_kv_import")
fs_kv_export = _wrap("fs_kv_export")
fs_kv_set_length = _wrap("fs_kv_set_length")
fs_prefill = _wrap("fs_prefill")
fs_decode_step = _wrap("fs_decode_step")
fs_forward_batch = _wrap("fs_forward_batch")
fs_greedy = _wrap("fs_greedy")
fs_sample = _wrap("fs_sample")
fs_generate = _wrap("fs_generate")
fs_debug_capture = _wrap("fs_debug_capture")
fs_debug_block = _wrap("fs_debug_block")
fs_debug_dequant_q8_0 = _wrap("fs_debug_dequant_q8_0")
fs_debug_trace = _wrap("fs_debug_trace")
fs_debug_wait_limit = _wrap("fs_debug_wait_limit")
fs_debug_decode_path = _wrap("fs_debug_decode_path")
fs_debug_decode_kernel = _wrap("fs_debug_decode_kernel")
fs_debug_lm_head = _wrap("fs_debug_lm_head")
fs_device_error = _wrap("fs_device_error")
fs_set_prefill_split = _wrap("fs_set_prefill_split")
fs_lm_head_argmax_noalloc = _wrap("fs_lm_head_argmax_noalloc")
fs_debug_kernel_launches = _wrap("fs_debug_kernel_launches")
fs_last_error_string = _wrap("fs_last_error_string")
fs_status_string = _wrap("fs_status_string")
