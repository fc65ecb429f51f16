"""Build libpagedattn.so in-tree with nvcc for sm_100a (static CUDA runtime, no torch extension).

    python -m pagedattention_paged_kv_attention_b200.build [--force] [-D NAME=VALUE ...] [--output PATH]

-D PA_TRACE --output libpagedattn_trace.so builds the timing-trace variant of the decode kernels (their
work is unchanged; they also write %globaltimer records into the workspace) under another name.

Each translation unit (.cu, and the host-only .cpp) is compiled in parallel, then linked into one shared library next to this
file. The library exports only the C ABI declared in include/*.h.
"""
import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(HERE, "libpagedattn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["pa_api.cu", "pa_attention_bf16.cu", "pa_attention_f16.cu", "pa_static_workspace.cu",
           "pa_prefill.cu", "pa_probe.cu", "pa_block_manager.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _stale(output, extra_defines):
    if not os.path.exists(output):
        return True
    mtime = os.path.getmtime(output)
    for d in (CSRC, INCLUDE):
        for name in os.listdir(d):
            if os.path.getmtime(os.path.join(d, name)) > mtime:
                return True
    return bool(extra_defines)


def build(force=False, defines=(), output=None, verbose=False):
    output = output or LIBRARY
    if not force and not _stale(output, defines):
        return output
    build_dir = os.path.join(HERE, "_build", "-".join(sorted(defines)) or "default")
    os.makedirs(build_dir, exist_ok=True)
    dflags = [f"-D{d}" for d in defines]

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.splitext(src)[0] + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *dflags, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
        return obj, r.stderr

    with concurrent.futures.ThreadPoolExecutor(len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    tmp = output + f".tmp{os.getpid()}"
    link = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *[o for o, _ in results], "-ldl"]
    r = subprocess.run(link, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, output)
    return output


if __name__ == "__main__":
    args = sys.argv[1:]
    defines = [args[i + 1] for i, a in enumerate(args) if a == "-D"]
    output = next((os.path.abspath(args[i + 1]) for i, a in enumerate(args) if a == "--output"), None)
    print(build(force="--force" in args, defines=defines, output=output, verbose="-v" in args))
