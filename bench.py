#!/usr/bin/env python3
"""Benchmark of libfs on the Qwen3-0.6B shape.

One step = one greedy generation job: prefill of an 8-token uniform-random
prompt, then 256 greedy decode steps at batch 1, ids kept on the device (the
next step's input is the previous step's argmax). ``value`` is decode
tokens/s over the whole job (prefill time included). Weights are seeded
random-init bf16 N(0, 0.02) (1.19 GB, larger than L2, so every step streams
them from HBM).

Also reported:
* ``roofline``: the decode forward against HBM bandwidth (algorithmic weight +
  KV bytes per decode step / measured step time);
* ``prefill``: a 2048-token prefill, tokens/s and TFLOP/s against bf16 peak;
* ``batched_decode``: batch 16 with 8192 pre-filled KV positions per sequence,
  tokens/s against HBM bandwidth (weights + KV bytes per step);
* ``q8_0_decode``: batch-1 decode with Q8_0 linear weights, tokens/s against
  HBM bandwidth (34 bytes per 32 linear weights);
* ``e2e``: the same job through ``fs_greedy`` with host buffers (prompt in,
  ids out, copies inside the timed region);
* ``cpu_baseline``: the CPU oracle on a bounded sample of the same job.

``--impl reference`` times the CPU oracle itself (the only reference this
workload has) on the same metric.

Multi-GPU (``--gpus N`` under torchrun): N independent replicas, no
collective in the data path; ``value`` sums the tokens of all ranks over the
slowest rank's time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

PROMPT = 8
DECODE_STEPS = 256
PREFILL_S = 2048
SEED = 1

# DRAM bytes (read + write) of one decode-kernel launch as an ncu capture
# measured them, with the capture's context length and date; None until the
# current decode kernel has been captured (the JSON line then reports null).
DECODE_TRAFFIC = {"bytes": 1_203_232_960, "context": 53, "taken": "2026-12-03"}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def decode_bytes(shape, ctx_lens, q8=False):
    """Algorithmic HBM bytes of one batch-1 decode step at each context length:
    every weight once (linear + tied embedding/LM head + norms) + the KV read
    (all positions incl. the new one) + the KV write of the new position.
    Q8_0 linear weights take 34 bytes per 32 (int8 codes + one fp16 scale)."""
    from dense_token_decode_b200.synth import LINEAR_NAMES, linear_shape
    n_lin = sum(a * b for a, b in (linear_shape(shape, n) for n in LINEAR_NAMES))
    lin = n_lin * 34 // 32 if q8 else n_lin * 2
    norms = (2 * shape.hidden + 2 * shape.head_dim) * 2
    weights = shape.n_layers * (lin + norms) + shape.vocab * shape.hidden * 2 + shape.hidden * 2
    kv_tok = shape.n_layers * 2 * shape.n_kv_heads * shape.head_dim * 2
    return [weights + kv_tok * c + kv_tok for c in ctx_lens], weights


def prefill_flops(shape, S):
    from dense_token_decode_b200.synth import LINEAR_NAMES, linear_shape
    lin = 2 * S * shape.n_layers * sum(a * b for a, b in (linear_shape(shape, n)
                                                          for n in LINEAR_NAMES))
    # causal attention: QK^T and PV over the S(S+1)/2 visible pairs, every query head
    attn = shape.n_layers * shape.n_q_heads * 2 * 2 * shape.head_dim * (S * (S + 1) // 2)
    head = 2 * shape.hidden * shape.vocab
    return lin + attn + head


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        else:
            self.lines = []

    def summary(self):
        sm, mx, reasons = [], None, set()
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time (the job's time): an all-reduce MAX over the
    process group (on the GPU under NCCL, on the host under gloo)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_this_rank: float) -> tuple[float, float]:
    """Whole-job tokens/s of N independent replicas: every rank's tokens over
    the slowest rank's time. Returns (value, max ms)."""
    ms_max = max_over_ranks(ms_this_rank, world)
    return tokens_per_rank * world / (ms_max / 1e3), ms_max


# --------------------------------------------------------------------------- CPU oracle

def host_cpu():
    """The host's logical core count and CPU model (for the CPU baseline)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count(), model


def oracle_decode_sample(shape, n_decode: int, n_warm: int = 0):
    """The CPU oracle (single BLAS thread) on the head of the same job: the
    8-token prompt prefill, n_warm untimed greedy decode steps, then n_decode
    timed ones. Returns (seconds per decode token, cores)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle
    from dense_token_decode_b200 import synth

    w = synth.model_weights(shape, SEED)

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    ow = {"embed": bits(w["embed"]), "final_norm": bits(w["final_norm"]),
          "layers": [{k: bits(v) for k, v in lw.items()} for lw in w["layers"]]}
    del w
    with threadpool_limits(1):
        orc = oracle.Qwen3Oracle(shape, ow)
        prompt = synth.token_ids(PROMPT, shape.vocab, seed=SEED).tolist()
        logits, _, cache = orc.forward(prompt)
        tok = oracle.greedy_select(logits)
        for _ in range(n_warm):
            logits, _, cache = orc.forward([tok], cache)
            tok = oracle.greedy_select(logits)
        t0 = time.perf_counter()
        for _ in range(n_decode):
            logits, _, cache = orc.forward([tok], cache)
            tok = oracle.greedy_select(logits)
        dt = time.perf_counter() - t0
    return dt / n_decode, 1


def run_reference(args, world, rank):
    if rank != 0:
        return
    from dense_token_decode_b200 import synth
    shape = synth.QWEN3_0P6B
    # Each step: one decode token of the job, by the oracle (warm-up steps untimed).
    per_tok, cores = oracle_decode_sample(shape, args.steps, args.warmup)
    value = 1.0 / per_tok
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_tok * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "host_cores": host_cpu()[0], "cpu_model": host_cpu()[1],
                         "sample": f"{args.steps} timed greedy decode steps after the 8-token "
                                   f"prompt and {args.warmup} untimed ones (fp64 numpy, one "
                                   f"BLAS thread)"},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# --------------------------------------------------------------------------- GPU

METRIC = "decode tok/s @bs1 Qwen3-0.6B shape (% HBM roofline); prefill tok/s (% tensor peak)"


def workload_config():
    return {"workload": "Qwen3-0.6B shape (28L, H1024, 16q/8kv x128, I3072, V151936, tied), "
                        "random-init bf16; 8-token prompt + 256 greedy decode steps at batch 1",
            "global_batch": 1, "seq_len": PROMPT + DECODE_STEPS, "parallelism": "replicas",
            "l2": "weights (1.19 GB) larger than L2: every step streams them from HBM"}


def run_ours(args, world, rank, local):
    import ctypes as C

    from dense_token_decode_b200 import abi, synth
    from dense_token_decode_b200.engine import Model

    dev = torch.device("cuda", local)
    shape = synth.QWEN3_0P6B
    w = synth.model_weights(shape, SEED)
    model = Model(shape, w, dev, max_pos=8192 + 256)
    del w
    kv = model.kv(1, PROMPT + DECODE_STEPS + 64)
    prompt = synth.token_ids(PROMPT, shape.vocab, seed=SEED).to(dev)
    gen = torch.zeros(DECODE_STEPS + 1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    dec_ev = []

    def job(record=False):
        kv.set_length(0, 0)
        model.prefill(kv, 0, prompt, None, gen[0:1])
        if record:
            a = torch.cuda.Event(enable_timing=True)
            a.record(stream)
        for i in range(DECODE_STEPS):
            model.decode_step(kv, [0], gen[i:i + 1], None, gen[i + 1:i + 2])
        if record:
            b = torch.cuda.Event(enable_timing=True)
            b.record(stream)
            dec_ev.append((a, b))

    for _ in range(args.warmup):
        job()
    torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    l0 = abi.fs_debug_kernel_launches()
    with ClockSampler(local) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            job(record=True)
        t1.record(stream)
        torch.cuda.synchronize(dev)
    launches = abi.fs_debug_kernel_launches() - l0
    barrier(world)
    ms = t0.elapsed_time(t1)
    value, ms_max = job_throughput(DECODE_STEPS * args.steps, world, ms)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_ev) / args.steps

    hbm, bf16, bf16_s, peak_src = peaks()
    ctx = [PROMPT + i + 1 for i in range(DECODE_STEPS)]  # context incl. the new position
    per_step, weight_bytes = decode_bytes(shape, ctx)
    step_s = dec_ms / 1e3 / DECODE_STEPS
    achieved = statistics.mean(per_step) / step_s / 1e9
    # the captured launch's traffic, moved to the job's mean context (KV grows by
    # one position's K and V per step)
    kv_tok = shape.n_layers * 2 * shape.n_kv_heads * shape.head_dim * 2
    traffic = None
    if DECODE_TRAFFIC is not None:
        traffic = DECODE_TRAFFIC["bytes"] + kv_tok * (statistics.mean(ctx)
                                                      - DECODE_TRAFFIC["context"])

    # End to end: fs_greedy with host buffers (prompt H2D, ids D2H inside the call).
    host_prompt = prompt.cpu().pin_memory()
    host_out = torch.zeros(DECODE_STEPS, dtype=torch.int32).pin_memory()
    n_out, why = C.c_int32(), C.c_int32()

    def e2e_job():
        kv.set_length(0, 0)
        abi.check(abi.fs_greedy(model.handle, kv.handle, 0, host_prompt.data_ptr(), PROMPT,
                                DECODE_STEPS, None, 0, host_out.data_ptr(), C.byref(n_out),
                                C.byref(why), stream.cuda_stream), "fs_greedy")

    for _ in range(max(1, args.warmup)):
        e2e_job()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_job()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_val, _ = job_throughput(DECODE_STEPS * args.steps, world, e0.elapsed_time(e1))
    assert n_out.value == DECODE_STEPS

    # Prefill of 2048 tokens.
    pre = None
    if not args.no_prefill:
        kvp = model.kv(1, PREFILL_S)
        ptoks = synth.token_ids(PREFILL_S, shape.vocab, seed=2).to(dev)
        am = torch.zeros(1, dtype=torch.int32, device=dev)

        def pjob():
            kvp.set_length(0, 0)
            model.prefill(kvp, 0, ptoks, None, am)

        for _ in range(2):
            pjob()
        torch.cuda.synchronize(dev)
        reps = 5
        p0 = torch.cuda.Event(enable_timing=True)
        p1 = torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        for _ in range(reps):
            pjob()
        p1.record(stream)
        torch.cuda.synchronize(dev)
        pms = p0.elapsed_time(p1) / reps
        flops = prefill_flops(shape, PREFILL_S)
        tf = flops / (pms / 1e3) / 1e12
        pre = {"value": PREFILL_S / (pms / 1e3), "unit": "tok/s", "ms": pms,
               "tflops": tf, "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16,
                                          "unit": "TFLOP/s", "frac": tf / bf16,
                                          "flops": flops, "peak_source": peak_src}}
        kvp.close()

    # Q8_0 decode at batch 1: the same job shape with Q8_0 linear weights
    # (embedding / LM head bf16), 256 greedy steps after the 8-token prompt.
    q8r = None
    if not args.no_q8:
        wq = synth.model_weights(shape, 4, "q8_0")
        mq = Model(shape, wq, dev, max_pos=1024)
        del wq
        QSTEPS = DECODE_STEPS
        kvq = mq.kv(1, PROMPT + QSTEPS + 16)
        qgen = torch.zeros(QSTEPS + 8, dtype=torch.int32, device=dev)
        qprompt = synth.token_ids(PROMPT, shape.vocab, seed=4).to(dev)

        def qjob(n):
            kvq.set_length(0, 0)
            mq.prefill(kvq, 0, qprompt, None, qgen[0:1])
            for i in range(n):
                mq.decode_step(kvq, [0], qgen[i:i + 1], None, qgen[i + 1:i + 2])

        qjob(8)
        qjob(8)
        torch.cuda.synchronize(dev)
        kvq.set_length(0, 0)
        mq.prefill(kvq, 0, qprompt, None, qgen[0:1])
        q0 = torch.cuda.Event(enable_timing=True)
        q1 = torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for i in range(QSTEPS):
            mq.decode_step(kvq, [0], qgen[i:i + 1], None, qgen[i + 1:i + 2])
        q1.record(stream)
        torch.cuda.synchronize(dev)
        qms = q0.elapsed_time(q1) / QSTEPS
        qbytes, _ = decode_bytes(shape, [PROMPT + i + 1 for i in range(QSTEPS)], q8=True)
        qach = statistics.mean(qbytes) / (qms / 1e3) / 1e9
        q8r = {"value": 1e3 / qms, "unit": "tok/s", "ms_per_step": qms,
               "workload": f"batch 1, Q8_0 linear weights, 8-token prompt + {QSTEPS} decode steps",
               "roofline": {"bound": "hbm", "achieved": qach, "peak": hbm, "unit": "GB/s",
                            "frac": qach / hbm, "bytes_per_step": statistics.mean(qbytes),
                            "peak_source": peak_src}}
        kvq.close()
        mq.close()

    # Batched decode: 16 sequences, each with 8192 pre-filled N(0,1) bf16 K/V
    # positions, 64 greedy steps (ids stay on the device).
    bat = None
    if not args.no_batched:
        B, CTX, BSTEPS = 16, 8192, 64
        kvb = model.kv(B, CTX + BSTEPS + 8)
        for q in range(B):
            for l in range(shape.n_layers):
                k, v = synth.prefilled_kv(shape, CTX, seed=3, seq=q, layer=l, device=dev)
                kvb.import_(q, l, 0, k, v)
        btok = synth.token_ids(B, shape.vocab, seed=3).to(dev)
        bgen = torch.zeros((BSTEPS + 1, B), dtype=torch.int32, device=dev)
        seqs = list(range(B))

        def reset_batch():
            torch.cuda.synchronize(dev)
            for q in range(B):
                kvb.set_length(q, CTX)
            bgen[0].copy_(btok)

        def bjob(n):
            for i in range(n):
                model.decode_step(kvb, seqs, bgen[i], None, bgen[i + 1])

        reset_batch()
        bjob(3)
        reset_batch()
        torch.cuda.synchronize(dev)
        b0 = torch.cuda.Event(enable_timing=True)
        b1 = torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        bjob(BSTEPS)
        b1.record(stream)
        torch.cuda.synchronize(dev)
        bms = b0.elapsed_time(b1) / BSTEPS
        kv_tok = shape.n_layers * 2 * shape.n_kv_heads * shape.head_dim * 2
        bbytes = weight_bytes + sum(kv_tok * (CTX + i + 1) + kv_tok
                                    for i in range(BSTEPS)) / BSTEPS * B
        bach = bbytes / (bms / 1e3) / 1e9
        bat = {"value": B / (bms / 1e3), "unit": "tok/s", "ms_per_step": bms,
               "workload": f"batch {B}, {CTX} pre-filled positions per sequence, "
                           f"{BSTEPS} greedy steps",
               "roofline": {"bound": "hbm", "achieved": bach, "peak": hbm, "unit": "GB/s",
                            "frac": bach / hbm, "bytes_per_step": bbytes,
                            "peak_source": peak_src}}
        kvb.close()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, cores = oracle_decode_sample(shape, args.cpu_steps)
        cpu = {"value": 1.0 / sec, "unit": "tok/s", "cores": cores, "kind": "oracle",
               "host_cores": host_cpu()[0], "cpu_model": host_cpu()[1],
               "sample": f"{args.cpu_steps} greedy decode steps after the 8-token prompt of "
                         f"the same job (fp64 numpy oracle, one BLAS thread)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "precision": "decode: bf16 (or Q8_0) weights widened in registers, fp32 FMA; "
                         "prefill: fp16 tensor-core operands (two terms where K/V are "
                         "rounded), fp32 accumulation; KV cache bf16",
            "config": workload_config(),
            "roofline": {"bound": "hbm", "kernel": "decode forward step", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": traffic,
                         "traffic_source": (None if DECODE_TRAFFIC is None else
                                            f"ncu dram bytes of one launch at context "
                                            f"{DECODE_TRAFFIC['context']}, taken "
                                            f"{DECODE_TRAFFIC['taken']}, moved to the mean "
                                            f"context"),
                         "bytes_per_step": statistics.mean(per_step),
                         "weight_bytes": weight_bytes, "step_us": step_s * 1e6,
                         "peak_source": peak_src},
            "e2e": {"value": e2e_val, "unit": "tok/s", "h2d_bytes_per_step": PROMPT * 4,
                    "d2h_bytes_per_step": DECODE_STEPS * 4},
            "gpu_launches": int(launches),
            "clocks": clocks.summary(),
            "prefill": pre,
            "batched_decode": bat,
            "q8_0_decode": q8r,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    kv.close()
    model.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-batched", action="store_true")
    ap.add_argument("--no-q8", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=16)
    args = ap.parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
