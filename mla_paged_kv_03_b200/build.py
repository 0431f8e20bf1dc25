"""Build libmla_b200.so in-tree with nvcc for sm_100a.

    python -m mla_paged_kv_03_b200.build [--force]

The build fails if ptxas reports more than SPILL_LIMIT bytes of register
spill stores in any kernel (the reference project's setup fails on any spill
[FlashMLA (AI Wiki), "Requirements and build"]; a few bytes in the fused and
sparse variants' rarely taken paths are tolerated here and reported).
"""
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmla_b200.so")
SOURCES = [os.path.join(CSRC, "mla_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + \
    [os.path.join(ROOT, "include", "mla.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SPILL_LIMIT = 64  # bytes of spill stores tolerated per kernel
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-v",
    "-shared",
]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False, out: str = None, defines=()) -> str:
    """Compile libmla_b200.so (or `out`, with extra -D `defines`)."""
    target = out or LIB
    if not force and not defines and out is None and not _stale():
        return LIB
    cmd = [NVCC] + FLAGS + [f"-D{d}" for d in defines] + \
        ["-I", os.path.join(ROOT, "include"), "-o", target] + SOURCES + ["-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    log = r.stdout + r.stderr
    if r.returncode != 0:
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed building libmla_b200.so")
    spills = [l for l in log.splitlines()
              if (m := re.search(r"(\d+) bytes spill stores", l)) and int(m.group(1)) > SPILL_LIMIT]
    if spills:
        if os.path.exists(target):
            os.remove(target)
        sys.stderr.write(log)
        raise RuntimeError("register spill in libmla_b200 kernels:\n" + "\n".join(spills))
    if verbose:
        sys.stderr.write(log)
    if out is None:
        with open(os.path.join(HERE, "ptxas_report.txt"), "w") as f:
            f.write(log)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
