"""Build step for libep_b200.so (nvcc, sm_100a only).

``python -m combine_ep_route_02_b200.build`` compiles every ``csrc/*.cu``
into ``combine_ep_route_02_b200/lib/libep_b200.so``.  The library links the
CUDA runtime statically, so it loads next to any PyTorch build.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libep_b200.so")
# the library the binding loads: LIB, or another build of it named by
# EP_B200_LIB (for example one installed elsewhere)
LOAD_LIB = os.environ.get("EP_B200_LIB") or LIB
HEADER = os.path.join(ROOT, "include", "ep.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                 "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.c")) + [HEADER]
    return any(os.path.getmtime(d) > t for d in deps)


def generate_tables(build_dir: str) -> None:
    """Writes silu_table.inc (the expert activation's SiLU table) into
    build_dir with the host generator csrc/gen_silu_table.c."""
    exe = os.path.join(build_dir, f"gen_silu_table.{os.getpid()}")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-o", exe,
                           os.path.join(CSRC, "gen_silu_table.c"), "-lm"])
    out = os.path.join(build_dir, "silu_table.inc")
    with open(out + ".tmp", "w") as f:
        subprocess.check_call([exe], stdout=f)
    os.replace(out + ".tmp", out)
    os.remove(exe)


# Per-file compiler options (none needed at present).
PER_FILE = {}

BUILD_DIR = os.path.join(PKG, "_build")


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    os.makedirs(BUILD_DIR, exist_ok=True)
    tag = f"{os.getpid()}"
    generate_tables(BUILD_DIR)
    procs, objs = [], []
    for src in sources():
        name = os.path.basename(src)
        obj = os.path.join(BUILD_DIR, name[:-3] + f".{tag}.o")
        cmd = [nvcc(), *ARCH, *COMPILE_FLAGS, *PER_FILE.get(name, []), *extra,
               "-I", BUILD_DIR, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        procs.append((subprocess.Popen(cmd), cmd))
        objs.append(obj)
    failed = [cmd for p, cmd in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    tmp = LIB + f".tmp{tag}"
    subprocess.check_call([nvcc(), *ARCH, "--shared", "-o", tmp, *objs])
    for o in objs:
        os.remove(o)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
