"""libfs: the forward pass of a dense Qwen3-class decoder (prefill and
KV-cached decode) as hand-written CUDA for B200 (sm_100a) behind a C ABI.

``abi`` holds the ctypes binding with the C names (fs_model_create, fs_kv_alloc,
fs_prefill, fs_decode_step, fs_greedy, ...); ``engine`` wraps them in small
handles that take torch tensors; ``synth`` draws the seeded synthetic inputs.
"""

from . import abi, synth  # noqa: F401
from .abi import (  # noqa: F401
    fs_debug_block,
    fs_debug_capture,
    fs_debug_dequant_q8_0,
    fs_debug_lm_head,
    fs_decode_step,
    fs_device_error,
    fs_greedy,
    fs_kv_alloc,
    fs_kv_export,
    fs_kv_free,
    fs_kv_import,
    fs_kv_length,
    fs_kv_reset,
    fs_kv_set_length,
    fs_last_error_string,
    fs_model_create,
    fs_model_destroy,
    fs_prefill,
    fs_set_prefill_split,
    fs_status_string,
)
from .engine import KV, Model  # noqa: F401
