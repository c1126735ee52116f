"""Build the CUDA library in-tree: fp8_scaled_matrix_b200/libfp8sm.so.

Every translation unit is compiled for sm_100a only
(-gencode arch=compute_100a,code=sm_100a), with the CUDA runtime linked
statically so the .so needs nothing but the driver at load time.  No fast
math: the quantizer's fp32 divisions and multiplies must stay IEEE.
"""
import concurrent.futures as cf
import fcntl
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libfp8sm.so")
BUILD_DIR = os.path.join(HERE, "_build")
SOURCES = ["capi.cu", "quantize.cu", "gemm.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return p


def _flags(verbose_ptxas: bool):
    f = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
                "-I", CSRC, "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(ROOT, "include", "fp8sm.h"))
    return files


def _up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    newest = max(os.path.getmtime(f) for f in _deps())
    return os.path.getmtime(LIB) >= newest


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile the library if it is missing or older than its sources.
    Several processes (one per GPU) may call this at once: an exclusive file
    lock serialises them, and the ones that wait find the library built."""
    if not force and _up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    with open(os.path.join(BUILD_DIR, ".lock"), "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        try:
            if not force and _up_to_date():
                return LIB
            return _build_locked(verbose_ptxas)
        finally:
            fcntl.flock(lock, fcntl.LOCK_UN)


def _build_locked(verbose_ptxas: bool) -> str:
    objs = []
    cmds = []
    for src in SOURCES:
        obj = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
        objs.append(obj)
        cmds.append([nvcc(), "-c", os.path.join(CSRC, src), "-o", obj] + _flags(verbose_ptxas))
    with cf.ThreadPoolExecutor(max_workers=len(cmds)) as ex:
        results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), cmds))
    for c, r in zip(cmds, results):
        if verbose_ptxas or r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed: " + " ".join(c))
    tmp = f"{LIB}.tmp{os.getpid()}"
    link = [nvcc(), "-shared", "-o", tmp] + objs + ARCH + [
        "-cudart", "static", "-Xcompiler", "-fPIC"]
    r = subprocess.run(link, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
