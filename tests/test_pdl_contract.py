"""Programmatic dependent launch contract, checked on the sources (CPU only).

A kernel started with launch_pdl may run while the kernel before it on the
stream is still running, so it must call pdl_wait() before it reads or writes
anything an earlier kernel touched. This test finds every kernel the sources
pass to launch_pdl and checks that its definition calls pdl_wait(), and that
nothing but weight loads (`load_w`) and index arithmetic comes before it.
"""

import pathlib
import re

CSRC = pathlib.Path(__file__).resolve().parents[1] / "dense_token_decode_b200" / "csrc"


def sources():
    return {p.name: p.read_text() for p in sorted(CSRC.glob("*.cu"))}


def kernel_body(src, name):
    """The body of `__global__ ... name(...) { ... }` (first definition)."""
    m = re.search(r"__global__[^;{]*?\b" + re.escape(name) + r"\s*\(", src)
    if not m:
        return None
    i = src.index("{", m.end())
    depth = 0
    for k in range(i, len(src)):
        if src[k] == "{":
            depth += 1
        elif src[k] == "}":
            depth -= 1
            if depth == 0:
                return src[i + 1:k]
    raise AssertionError(f"unbalanced braces in {name}")


def launched_kernels(srcs):
    names = set()
    for text in srcs.values():
        for m in re.finditer(r"launch_pdl\(\s*([A-Za-z0-9_:]+)", text):
            names.add(m.group(1).split("::")[-1])
    return names


def test_every_dependent_launch_waits():
    srcs = sources()
    names = launched_kernels(srcs)
    assert {"gemv_mma_kernel", "rmsnorm_kernel", "gemm_tc_kernel",
            "attention_tc_kernel"} <= names
    for name in sorted(names):
        bodies = [b for b in (kernel_body(t, name) for t in srcs.values()) if b]
        assert bodies, f"no definition of {name}"
        body = bodies[0]
        assert "pdl_wait()" in body, f"{name} is launched dependently but never waits"
        before = body[:body.index("pdl_wait()")]
        # Before the wait: weights only (the GEMV's load_w), no shared-memory
        # staging, no global stores or atomics.
        assert "atomicAdd" not in before and "__syncthreads" not in before, name
        assert not re.search(r"\b(xs|hs|zero|out)\s*\[[^;]*\]\s*=[^=]", before), name
        assert not re.search(r"\bout\s*\+", before), name
