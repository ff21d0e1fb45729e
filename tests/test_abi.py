"""The C-ABI library loads and exports every symbol include/fs.h declares, and
host-side argument checks fail cleanly without touching a GPU."""

import ctypes as C
import os
import re

import pytest

from dense_token_decode_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "fs.h")).read()
    return sorted(set(re.findall(r"\b(fs_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(abi.SIGNATURES)


def test_library_exports_every_declared_symbol():
    lib = abi.load()
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings():
    assert abi.fs_status_string(abi.FS_ERR_TOKEN) == b"FS_ERR_TOKEN"
    assert abi.fs_status_string(0) == b"FS_OK"


def test_null_arguments_are_rejected_on_the_host():
    out = C.c_void_p(123)
    assert abi.fs_model_create(None, None, C.byref(out)) == abi.FS_ERR_NULL
    assert out.value is None
    assert abi.fs_kv_alloc(None, 1, 1, C.byref(out)) == abi.FS_ERR_NULL
    assert abi.fs_prefill(None, None, 0, None, 1, None, None, None) == abi.FS_ERR_NULL
    assert abi.fs_debug_dequant_q8_0(None, None, 4, 33, None, None) == abi.FS_ERR_INVALID
    n, r = C.c_int32(), C.c_int32()
    assert abi.fs_greedy(None, None, 0, None, 0, 0, None, 0, None, C.byref(n), C.byref(r),
                         None) == abi.FS_ERR_NULL
    abi.fs_model_destroy(None)
    abi.fs_kv_free(None)


def test_bad_configs_are_rejected_before_any_device_work():
    from dense_token_decode_b200 import engine, synth
    w = abi.fs_weights(None, None, None)
    out = C.c_void_p()
    bad = [
        dict(n_q_heads=3),            # 3 % 2 kv heads
        dict(head_dim=96),            # unsupported head_dim
        dict(hidden=100),             # not a multiple of 64
        dict(n_layers=0),
    ]
    for kw in bad:
        shape = synth.ModelShape(**{**synth.TINY.__dict__, **kw})
        cfg = engine.make_config(shape)
        st = abi.fs_model_create(C.byref(cfg), C.byref(w), C.byref(out))
        assert st in (abi.FS_ERR_INVALID, abi.FS_ERR_UNSUPPORTED), (kw, st)
    cfg = engine.make_config(synth.TINY)
    assert abi.fs_model_create(C.byref(cfg), C.byref(w), C.byref(out)) == abi.FS_ERR_NULL


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(abi, "_lib", None)
    monkeypatch.setattr(abi, "_LIB_PATH", "/nonexistent/libfs.so")
    with pytest.raises(abi.LibraryMissing):
        abi.load()
