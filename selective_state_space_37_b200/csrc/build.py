"""Build libselscan.so in-tree for sm_100a with nvcc (no GPU needed).

    python -m selective_state_space_37_b200.csrc.build [--force] [--verbose]

The CUDA runtime is linked statically so the library loads in any process
(with or without torch) on a machine with a CUDA 12.9-capable driver.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
LIB = os.path.join(HERE, "libselscan.so")
SOURCES = ["selscan.cu"]
HEADERS = ["common.cuh", "cp_async.cuh", "fwd.cuh", "ssd_tc.cuh", "bwd.cuh", "step.cuh", "block.cuh", "ssd.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
    "-lcublas", "-Xlinker", "-rpath", "-Xlinker", "/usr/local/cuda/lib64",
]


def _inputs():
    files = [os.path.join(HERE, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "selscan.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, out: str = LIB, defines=()) -> str:
    """Compile the library to `out`; `defines` are extra -D preprocessor
    definitions passed to nvcc (e.g. for a differently configured copy built
    next to the in-tree one and loaded through SELSCAN_LIB)."""
    if not force and out == LIB and not defines and up_to_date():
        return out
    cmd = [NVCC, *NVCC_FLAGS] + [f"-D{d}" for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-shared", "-o", out + ".tmp"] + [os.path.join(HERE, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    defs = [a[2:] for a in sys.argv[1:] if a.startswith("-D")]
    outs = [a.split("=", 1)[1] for a in sys.argv[1:] if a.startswith("--out=")]
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                out=outs[0] if outs else LIB, defines=defs))
