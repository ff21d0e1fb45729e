"""Per-phase timeline of one persistent decode step (fs_debug_trace).

    python -m dense_token_decode_b200.trace [--fmt bf16|q8_0] [--context N]

Builds the Qwen3-0.6B shape with seeded random weights, decodes up to the
given context, arms the trace for one step and prints, per phase slot, the
earliest / median / latest CTA timestamp relative to the start of the layer
(median over the middle layers), then the mean step time of 100 untraced
steps. Slot meanings are those documented with fs_debug_trace in fs.h.
"""

from __future__ import annotations

import argparse

import numpy as np
import torch

from . import abi, synth
from .engine import Model

SLOTS = [(0, "QKV phase begins"), (1, "QKV input complete"), (2, "QKV rows done"),
         (3, "attention phase begins"), (4, "q/k/v ready"), (5, "attention done"),
         (6, "O share added"), (7, "MLP phase begins"), (8, "MLP input complete"),
         (9, "gate/up done"), (10, "down share added")]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmt", default="bf16", choices=["bf16", "q8_0"])
    ap.add_argument("--context", type=int, default=100)
    args = ap.parse_args()
    dev = "cuda:0"
    shape = synth.QWEN3_0P6B
    m = Model(shape, synth.model_weights(shape, 1, args.fmt), dev, max_pos=4096)
    n = args.context
    kv = m.kv(1, n + 128)
    prompt = synth.token_ids(8, shape.vocab, seed=1).to(dev)
    gen = torch.zeros(n + 128, dtype=torch.int32, device=dev)
    m.prefill(kv, 0, prompt, None, gen[0:1])
    for i in range(n):
        m.decode_step(kv, [0], gen[i:i + 1], None, gen[i + 1:i + 2])
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    L = shape.n_layers
    buf = torch.zeros((sms * (L + 1), 16), dtype=torch.int64, device=dev)
    abi.check(abi.fs_debug_trace(m.handle, buf.data_ptr()), "fs_debug_trace")
    m.decode_step(kv, [0], gen[n:n + 1], None, gen[n + 1:n + 2])
    torch.cuda.synchronize()
    raw = buf.cpu().numpy().astype(np.float64)
    t = raw[: sms * (L + 1)].reshape(sms, L + 1, 16)
    t = np.where(t > 0, t / 1000.0, np.nan)  # us
    print(f"context {n + 8}; us from the first QKV start of the layer, median of layers 3..{L - 3}")
    print(f"{'slot':34s} {'first':>7s} {'median':>7s} {'last':>7s}")
    for k, name in SLOTS:
        rows = []
        for l in range(3, L - 2):
            col = t[:, l, k]
            if np.isnan(col).all():
                continue
            base = np.nanmin(t[:, l, 0])
            rows.append((np.nanmin(col) - base, np.nanmedian(col) - base, np.nanmax(col) - base))
        if rows:
            a = np.median(np.array(rows), axis=0)
            print(f"{name:34s} {a[0]:7.2f} {a[1]:7.2f} {a[2]:7.2f}")
    ends = np.nanmax(t[:, :L, 10], axis=0)
    total = np.nanmax(t[:, L, 4]) - np.nanmin(t[:, 0, 0])
    print(f"layer time (median) {np.median(np.diff(ends)):.2f} us; tail (final norm, LM head, "
          f"greedy) {np.nanmax(t[:, L, 4]) - ends[-1]:.2f} us; whole step in the kernel "
          f"{total:.1f} us")
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n + 1, n + 101):
        m.decode_step(kv, [0], gen[i:i + 1], None, gen[i + 1:i + 2])
    e1.record()
    torch.cuda.synchronize()
    print(f"mean step {e0.elapsed_time(e1) * 1000 / 100:.1f} us over 100 untraced steps; "
          f"device error {m.device_error()}")
    m.close()


if __name__ == "__main__":
    main()
