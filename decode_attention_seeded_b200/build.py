"""Build libtq.so in-tree with nvcc for sm_100a (no GPU needed to build).

The decode and prefill kernel templates are instantiated once per (key bits,
value bits) pair in csrc/tq_inst.cu; the build compiles that file once per pair
and the other sources once, in parallel, then links the shared library.
"""

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
HEADERS = [os.path.join(ROOT, "include", "tq.h"), os.path.join(CSRC, "tq_internal.h"),
           os.path.join(CSRC, "tq_kernels.cuh")]
SOURCES = [os.path.join(CSRC, f) for f in ("tq_host.cpp", "tq_kernels.cu", "tq_inst.cu")]
BITS = [(2, 2), (2, 3), (2, 4), (3, 2), (3, 3), (3, 4), (4, 2), (4, 3), (4, 4), (8, 2), (8, 3), (8, 4)]
LIB = os.path.join(HERE, "libtq.so")
OBJ_DIR = os.path.join(ROOT, "_build", "obj")


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in SOURCES + HEADERS + [os.path.abspath(__file__)])


def _units():
    """(source, object, extra flags) of every compilation."""
    u = [(os.path.join(CSRC, "tq_host.cpp"), os.path.join(OBJ_DIR, "tq_host.o"), []),
         (os.path.join(CSRC, "tq_kernels.cu"), os.path.join(OBJ_DIR, "tq_kernels.o"), [])]
    for bk, bv in BITS:
        u.append((os.path.join(CSRC, "tq_inst.cu"), os.path.join(OBJ_DIR, f"tq_inst_{bk}_{bv}.o"),
                  [f"-DTQ_BK={bk}", f"-DTQ_BV={bv}"]))
    return u


def _compile(nvcc, src, obj, extra, verbose):
    cmd = [nvcc, "-std=c++17", "-O3", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-diag-suppress", "177",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    return src, extra, res


def build(force: bool = False, verbose: bool = False, jobs: int = 0) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = nvcc_path()
    os.makedirs(OBJ_DIR, exist_ok=True)
    units = _units()
    jobs = jobs or max(1, min(len(units), os.cpu_count() or 1))
    log = []
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        for src, extra, res in ex.map(lambda u: _compile(nvcc, *u, verbose), units):
            if res.returncode != 0:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)} {' '.join(extra)}:\n"
                                   + res.stdout + res.stderr)
            log.append(res.stderr)
    link = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
            *[obj for _, obj, _ in units], "-o", LIB + ".tmp"]
    res = subprocess.run(link, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("link failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write("".join(log))
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
