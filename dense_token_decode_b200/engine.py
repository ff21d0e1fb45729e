"""Thin Python handles over the C ABI: torch allocates device memory and
hands pointers and the current stream to libfs; nothing is computed here."""

from __future__ import annotations

import ctypes as C

import torch

from . import abi
from .synth import LINEAR_NAMES, NORM_NAMES, ModelShape


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def make_config(shape: ModelShape, weight_format: int = abi.FS_WEIGHT_BF16,
                max_pos: int | None = None) -> abi.fs_config:
    return abi.fs_config(shape.n_layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads,
                         shape.head_dim, shape.ffn, shape.vocab, shape.rms_eps, shape.rope_theta,
                         max_pos if max_pos is not None else shape.max_pos, weight_format)


class Model:
    """A libfs model over device copies of ``synth.model_weights`` tensors."""

    def __init__(self, shape: ModelShape, weights: dict, device="cuda:0", max_pos=None):
        self.shape = shape
        self.device = torch.device(device)
        q8 = isinstance(weights["layers"][0]["wq"], tuple)
        self.weight_format = abi.FS_WEIGHT_Q8_0 if q8 else abi.FS_WEIGHT_BF16
        dev = lambda t: t.to(self.device, non_blocking=False).contiguous()
        self._keep = []
        self.embed = dev(weights["embed"])
        self.final_norm = dev(weights["final_norm"])
        self._keep += [self.embed, self.final_norm]
        layer_structs = (abi.fs_layer_weights * shape.n_layers)()
        for l, lw in enumerate(weights["layers"]):
            s = layer_structs[l]
            for name in LINEAR_NAMES:
                w = lw[name]
                if isinstance(w, tuple):
                    codes, scales = dev(w[0]), dev(w[1])
                    self._keep += [codes, scales]
                    setattr(s, name, abi.fs_linear(codes.data_ptr(), scales.data_ptr()))
                else:
                    wd = dev(w)
                    self._keep.append(wd)
                    setattr(s, name, abi.fs_linear(wd.data_ptr(), None))
            for name in NORM_NAMES:
                g = dev(lw[name])
                self._keep.append(g)
                setattr(s, name, g.data_ptr())
        self._layers = layer_structs
        self.cfg = make_config(shape, self.weight_format, max_pos)
        self.fs_weights = abi.fs_weights(self.embed.data_ptr(), self.final_norm.data_ptr(),
                                         layer_structs)
        h = C.c_void_p()
        torch.cuda.synchronize(self.device)
        abi.check(abi.fs_model_create(C.byref(self.cfg), C.byref(self.fs_weights), C.byref(h)),
                  "fs_model_create")
        self.handle = h

    def close(self):
        if self.handle:
            torch.cuda.synchronize(self.device)
            abi.fs_model_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def kv(self, max_seqs: int, max_tokens: int) -> "KV":
        return KV(self, max_seqs, max_tokens)

    def prefill(self, kv: "KV", seq: int, tokens: torch.Tensor, logits=None, argmax=None,
                stream=None):
        abi.check(abi.fs_prefill(self.handle, kv.handle, seq, _ptr(tokens), tokens.numel(),
                                 _ptr(logits), _ptr(argmax), _stream(stream)), "fs_prefill")

    def decode_step(self, kv: "KV", seqs, tokens: torch.Tensor, logits=None, argmax=None,
                    stream=None):
        seq_arr = (C.c_int32 * len(seqs))(*seqs)
        abi.check(abi.fs_decode_step(self.handle, kv.handle, seq_arr, _ptr(tokens), len(seqs),
                                     _ptr(logits), _ptr(argmax), _stream(stream)),
                  "fs_decode_step")

    def forward_batch(self, kv: "KV", segments, logits=None, argmax=None, stream=None):
        """fs_forward_batch: ``segments`` is a list of (seq, token list)."""
        seqs = (C.c_int32 * len(segments))(*[q for q, _ in segments])
        lens = (C.c_int32 * len(segments))(*[len(t) for _, t in segments])
        flat = [t for _, ts in segments for t in ts]
        toks = (C.c_int32 * len(flat))(*flat)
        abi.check(abi.fs_forward_batch(self.handle, kv.handle, seqs, lens, len(segments),
                                       C.cast(toks, C.c_void_p), _ptr(logits), _ptr(argmax),
                                       _stream(stream)), "fs_forward_batch")

    def greedy(self, kv: "KV", seq: int, prompt, max_new: int, eos=(), out=None, stream=None):
        """Returns (ids list, stop reason). ``prompt``/``out`` may be host or device."""
        if not isinstance(prompt, torch.Tensor):
            prompt = torch.tensor(list(prompt), dtype=torch.int32)
        if out is None:
            out = torch.empty(max(max_new, 1), dtype=torch.int32)
        eos_arr = (C.c_int32 * max(len(eos), 1))(*eos)
        n_out, why = C.c_int32(0), C.c_int32(0)
        abi.check(abi.fs_greedy(self.handle, kv.handle, seq, _ptr(prompt), prompt.numel(), max_new,
                                eos_arr, len(eos), _ptr(out), C.byref(n_out), C.byref(why),
                                _stream(stream)), "fs_greedy")
        return out[: n_out.value].tolist(), why.value

    def generate(self, kv: "KV", seq: int, prompt, max_new: int, temperature: float,
                 top_k: int = 0, top_p: float = 1.0, seed: int = 0, eos=(), out=None,
                 stream=None):
        """fs_generate: like greedy() with seeded sampling. Returns (ids, reason)."""
        if not isinstance(prompt, torch.Tensor):
            prompt = torch.tensor(list(prompt), dtype=torch.int32)
        if out is None:
            out = torch.empty(max(max_new, 1), dtype=torch.int32)
        eos_arr = (C.c_int32 * max(len(eos), 1))(*eos)
        n_out, why = C.c_int32(0), C.c_int32(0)
        abi.check(abi.fs_generate(self.handle, kv.handle, seq, _ptr(prompt), prompt.numel(),
                                  max_new, eos_arr, len(eos), temperature, top_k, top_p, seed,
                                  _ptr(out), C.byref(n_out), C.byref(why), _stream(stream)),
                  "fs_generate")
        return out[: n_out.value].tolist(), why.value

    def sample(self, logits: torch.Tensor, temperature: float, top_k: int = 0,
               top_p: float = 1.0, seed: int = 0, step: int = 0, out=None, stream=None):
        """fs_sample on device logits [rows, V]; returns the int32 ids tensor."""
        rows = 1 if logits.dim() == 1 else logits.shape[0]
        if out is None:
            out = torch.empty(rows, dtype=torch.int32, device=logits.device)
        abi.check(abi.fs_sample(self.handle, logits.data_ptr(), rows, temperature, top_k, top_p,
                                seed, step, out.data_ptr(), _stream(stream)), "fs_sample")
        return out

    def capture(self, hidden: torch.Tensor | None, max_rows: int = 0):
        abi.check(abi.fs_debug_capture(self.handle, _ptr(hidden), max_rows), "fs_debug_capture")

    def block(self, kv: "KV", seq: int, layer: int, h_in: torch.Tensor, stream=None):
        """Run one block alone (fs_debug_block); returns h_out."""
        h_out = torch.empty_like(h_in)
        abi.check(abi.fs_debug_block(self.handle, kv.handle, seq, layer, h_in.data_ptr(),
                                     h_in.shape[0], h_out.data_ptr(), _stream(stream)),
                  "fs_debug_block")
        return h_out

    def lm_head(self, x: torch.Tensor, logits=None, argmax=None, stream=None):
        abi.check(abi.fs_debug_lm_head(self.handle, _ptr(x), x.shape[0], _ptr(logits),
                                       _ptr(argmax), _stream(stream)), "fs_debug_lm_head")

    def device_error(self) -> int:
        code = C.c_int32(0)
        abi.check(abi.fs_device_error(self.handle, C.byref(code)), "fs_device_error")
        return code.value

    def wait_limit(self, wait_ns: int, withhold_layer: int = -1):
        abi.check(abi.fs_debug_wait_limit(self.handle, wait_ns, withhold_layer),
                  "fs_debug_wait_limit")

    def decode_path(self, path: int):
        """0 auto, 1 cooperative, 2 general sequence, 3 row-split, 4 cluster kernel."""
        abi.check(abi.fs_debug_decode_path(self.handle, path), "fs_debug_decode_path")

    def decode_kernel(self, batch: int = 1) -> int:
        """3 row-split kernel, 2 cluster kernel, 1 cooperative kernel, 0 general sequence."""
        kind = C.c_int32(0)
        abi.check(abi.fs_debug_decode_kernel(self.handle, batch, C.byref(kind)),
                  "fs_debug_decode_kernel")
        return kind.value

    def set_prefill_split(self, split: int):
        abi.check(abi.fs_set_prefill_split(self.handle, split), "fs_set_prefill_split")


class KV:
    def __init__(self, model: Model, max_seqs: int, max_tokens: int):
        self.model = model
        h = C.c_void_p()
        abi.check(abi.fs_kv_alloc(model.handle, max_seqs, max_tokens, C.byref(h)), "fs_kv_alloc")
        self.handle = h

    def close(self):
        if self.handle:
            torch.cuda.synchronize(self.model.device)
            abi.fs_kv_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def length(self, seq: int) -> int:
        n = C.c_int32(0)
        abi.check(abi.fs_kv_length(self.handle, seq, C.byref(n)), "fs_kv_length")
        return n.value

    def reset(self, seq: int):
        abi.check(abi.fs_kv_reset(self.handle, seq), "fs_kv_reset")

    def set_length(self, seq: int, n: int):
        abi.check(abi.fs_kv_set_length(self.handle, seq, n), "fs_kv_set_length")

    def import_(self, seq: int, layer: int, pos0: int, k: torch.Tensor, v: torch.Tensor,
                stream=None):
        abi.check(abi.fs_kv_import(self.handle, seq, layer, pos0, k.shape[0], k.data_ptr(),
                                   v.data_ptr(), _stream(stream)), "fs_kv_import")

    def export(self, seq: int, layer: int, pos0: int, n: int, stream=None):
        s = self.model.shape
        k = torch.empty((n, s.n_kv_heads, s.head_dim), dtype=torch.bfloat16, device=self.model.device)
        v = torch.empty_like(k)
        abi.check(abi.fs_kv_export(self.handle, seq, layer, pos0, n, k.data_ptr(), v.data_ptr(),
                                   _stream(stream)), "fs_kv_export")
        return k, v
