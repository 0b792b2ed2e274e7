"""Every kernel launched with programmatic dependent launch (launch_chained) may
start before the kernel ahead of it on the stream has finished, so its first
statement must be chain_wait(): it is then ordered after everything that kernel
wrote. This reads the CUDA sources (no GPU)."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gaussian_splatting_differentiable_rasteriser_b200", "csrc")


def sources():
    out = {}
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name)) as f:
                out[name] = f.read()
    return out


def kernel_body_start(text, kernel):
    """The first statement of __global__ function `kernel` in `text`, or None."""
    m = re.search(r"__global__\s+void[^;{]*?\b" + re.escape(kernel) + r"\s*\(", text)
    if not m:
        return None
    i, depth = m.end(), 1
    while depth:
        depth += {"(": 1, ")": -1}.get(text[i], 0)
        i += 1
    body = text[text.index("{", i) + 1:]
    return body.lstrip().split(";", 1)[0].strip()


def test_every_chained_kernel_waits_first():
    src = sources()
    launched = set()
    for text in src.values():
        for m in re.finditer(r"launch_chained\(\s*([A-Za-z_][A-Za-z_0-9]*)", text):
            if m.group(1) != "void":  # the helper's own declaration
                launched.add(m.group(1))
    assert "preprocess_kernel" in launched and "blend_backward_kernel" in launched
    assert len(launched) >= 15
    for kernel in sorted(launched):
        firsts = [kernel_body_start(text, kernel) for text in src.values()]
        firsts = [f for f in firsts if f is not None]
        assert firsts, f"no definition of {kernel}"
        for f in firsts:
            assert f == "chain_wait()", f"{kernel} starts with {f!r}, not chain_wait()"


def test_the_helper_waits_before_it_releases():
    text = sources()["gs_kernels.cuh"]
    assert "griddepcontrol.wait" in text and "griddepcontrol.launch_dependents" in text
    assert "cudaLaunchAttributeProgrammaticStreamSerialization" in text
