"""Source-level rules of the CUDA library that no CPU run can exercise (CPU, reads the sources).

Kernels launched with programmatic stream serialisation (pa_host::launch_overlapped) may be scheduled
while the previous kernel in the stream still runs, so each of them must execute
grid_dependency_wait() before its first global-memory access. This test finds every such launch,
resolves the kernel it launches, and checks that the kernel body waits, and that nothing before the
wait reads or writes global memory (no __ldg, atomics, TMA or bulk copies, or subscripted global
pointers).
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "pagedattention_paged_kv_attention_b200", "csrc")

GLOBAL_ACCESS = re.compile(r"__ldg\(|atomic[A-Z]|\btma_load|cp\.async|\bargs\.\w+\s*\[|"
                           r"\b(?:block_mapping|slot_mapping|context_lens|block_tables|key|value)\s*\[")


def sources():
    return {n: open(os.path.join(CSRC, n)).read() for n in sorted(os.listdir(CSRC))
            if n.endswith((".cu", ".cuh", ".h"))}


def launched_kernels(srcs):
    names = set()
    for text in srcs.values():
        for m in re.finditer(r"launch_overlapped\(\s*([\w:<>, ]+?)\s*,\s*dim3", text):
            target = m.group(1)
            if target == "kernel":  # `auto kernel = NAME<...>;` earlier in the same function
                prior = re.findall(r"auto kernel = ([\w:]+)", text[:m.start()])
                target = prior[-1]
            names.add(re.sub(r"<.*", "", target).split("::")[-1])
    return names


def kernel_body(srcs, name):
    for text in srcs.values():
        m = re.search(r"__global__[^;{]*?\b" + name + r"\s*\(", text)
        if not m:
            continue
        start = text.index("{", m.end())
        depth = 0
        for i in range(start, len(text)):
            depth += {"{": 1, "}": -1}.get(text[i], 0)
            if depth == 0:
                return text[start + 1:i]
    raise AssertionError(f"no __global__ definition of {name}")


def test_overlapped_launches_wait_before_global_access():
    srcs = sources()
    names = launched_kernels(srcs)
    assert {"paged_attention_main", "paged_attention_reduce", "reshape_and_cache_kernel",
            "copy_blocks_kernel"} <= names, names
    for name in names:
        body = kernel_body(srcs, name)
        assert "grid_dependency_wait();" in body, f"{name} is launched overlapped but never waits"
        before = body[:body.index("grid_dependency_wait();")]
        hit = GLOBAL_ACCESS.search(before)
        assert hit is None, f"{name} touches global memory before its wait: {hit.group(0)!r}"


def test_rule_catches_an_access_before_the_wait():
    body = "const int64_t src = block_mapping[2 * pair];\n  grid_dependency_wait();"
    assert GLOBAL_ACCESS.search(body[:body.index("grid_dependency_wait();")])
