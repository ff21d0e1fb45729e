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

SLOTS = {
    # row-split kernel
    3: [(0, "QKV phase begins"), (1, "QKV input loaded"), (8, "QKV rows done"),
        (12, "attention item begins"), (2, "q/k/v loaded"), (13, "q/k normed, roped, K/V appended"),
        (14, "item's keys done"), (15, "warps merged"), (9, "attention merged"),
        (3, "O phase begins"), (4, "O input loaded"), (10, "gate/up phase begins"),
        (5, "gate/up input loaded"), (11, "down phase begins"), (6, "down input loaded"),
        (7, "block done")],
    # cooperative kernel
    1: [(0, "QKV phase begins"), (11, "QKV input slice reduced"), (1, "QKV input loaded"),
        (2, "QKV rows done"), (3, "attention phase begins"), (4, "q/k/v ready"),
        (13, "attention keys done"), (5, "attention merged"), (6, "O share added"),
        (7, "MLP phase begins"), (12, "MLP input slice reduced"), (8, "MLP input loaded"),
        (9, "gate/up done"), (10, "down share added")],
    # cluster kernel
    2: [(0, "block begins"), (1, "block input exchanged"), (2, "QKV rows done"),
        (3, "q/k/v exchanged, normed, rotated"), (4, "keys done, states sent"),
        (5, "attention merged and exchanged"), (6, "O shares published"),
        (7, "MLP input exchanged"), (8, "gate/up + SwiGLU done"),
        (9, "activations exchanged"), (10, "down shares published")],
}
HOPS = {
    3: [("QKV rows -> q/k/v loaded", 8, 2, 0), ("attention merged -> O input loaded", 9, 4, 0),
        ("block done -> next QKV input loaded", 7, 1, 1)],
    1: [("QKV rows -> q/k/v ready", 2, 4, 0), ("O shares -> MLP slice reduced", 6, 12, 0),
        ("down shares -> next QKV slice reduced", 10, 11, 1)],
    2: [("O shares -> MLP input exchanged", 6, 7, 0),
        ("down shares -> next block input exchanged", 10, 1, 1)],
}


def to_us(raw, sms, L):
    """Per-CTA cycle stamps -> us on a common time base: each CTA's stamps are
    placed with its own (globaltimer, clock) pairs taken at start and end."""
    t = raw[: sms * (L + 1)].reshape(sms, L + 1, 16).astype(np.float64)
    g0, c0, g1, c1 = (t[:, L, i] for i in (12, 13, 14, 15))
    ghz = (c1 - c0) / np.maximum(g1 - g0, 1.0)  # cycles per ns
    out = np.full_like(t, np.nan)
    ok = t > 0
    for c in range(sms):
        if ghz[c] <= 0:
            continue
        out[c] = (g0[c] + (t[c] - c0[c]) / ghz[c]) / 1000.0
    out[~ok] = np.nan
    out[:, L, 12:] = np.nan
    return out, float(np.median(ghz[ghz > 0]))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmt", default="bf16", choices=["bf16", "q8_0"])
    ap.add_argument("--context", type=int, default=100)
    ap.add_argument("--dump", default=None, help="save the raw stamps (.npy) to this path")
    ap.add_argument("--path", type=int, default=0, choices=[0, 1, 3, 4],
                    help="0 the default decode path, 1 the cooperative kernel, "
                         "3 the row-split kernel, 4 the cluster kernel")
    args = ap.parse_args()
    dev = "cuda:0"
    shape = synth.QWEN3_0P6B
    m = Model(shape, synth.model_weights(shape, 1, args.fmt), dev, max_pos=4096)
    m.decode_path(args.path)
    kind = m.decode_kernel(1)
    print("kernel:", {3: "row-split", 2: "cluster", 1: "cooperative", 0: "general"}[kind])
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
    if kind in SLOTS:
        raw = buf.cpu().numpy()
        if args.dump:
            np.save(args.dump, raw)
        t, ghz = to_us(raw, sms, L)
        print(f"context {n + 8}; SM clock {ghz:.3f} GHz; us from the first QKV start of the layer, "
              f"median of layers 3..{L - 3}")
        print(f"{'slot':34s} {'first':>7s} {'median':>7s} {'last':>7s}")
        # the tail row's slots 12..15 hold the start / end pairs, not phases
        for k, name in SLOTS.get(kind, []):
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
        # hand-offs: the last producer of a phase's input to the median consumer
        for name, k_from, k_to, dl in HOPS.get(kind, []):
            v = [np.nanmedian(t[:, l + dl, k_to]) - np.nanmax(t[:, l, k_from]) for l in range(3, L - 2)]
            print(f"hand-off {name:40s} {np.median(v):6.2f} us")
        end_slot, tail_slot = (7, 7) if kind == 3 else (10, 4)
        ends = np.nanmax(t[:, :L, end_slot], axis=0)
        total = np.nanmax(t[:, L, tail_slot]) - np.nanmin(t[:, 0, 0])
        print(f"layer time (median) {np.median(np.diff(ends)):.2f} us; tail (final norm, LM head, "
              f"greedy) {np.nanmax(t[:, L, tail_slot]) - ends[-1]:.2f} us; whole step in the "
              f"kernel {total:.1f} us")
    else:
        print("(no phase timeline for the general kernel sequence)")
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
