"""Build ``libssm_b200.so`` (the C-ABI selective-scan library) for sm_100a with nvcc.

The library is built in-tree next to this file so that it travels with the source tree.
Run ``python -m selective_state_space_23_b200.build`` (or ``build()`` from Python).
"""
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libssm_b200.so")
SOURCES = ["ssm_api.cu", "ssm_fwd.cu", "ssm_fwd_bf16.cu", "ssm_fwd_f32.cu", "ssm_fwd_rev_bf16.cu",
           "ssm_fwd_rev_f32.cu", "ssm_fwd_lane_bf16.cu", "ssm_fwd_lane_f32.cu", "ssm_bwd.cu", "ssm_bwd_hist.cu", "ssm_pcbc.cu", "ssm_ssd.cu", "ssm_decode.cu", "ssm_noalloc.cu", "ssm_host.cu",
           "ssm_strided.cu", "ssm_slices.cu", "ssm_ssd_bwd.cu"]
HEADERS = ["ssm_device.cuh", "ssm_kernels.h", "ssm_rows.cuh", "ssm_fwd_impl.cuh", "ssm_fwd_lane.cuh", "ssm_mma.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I" + os.path.join(ROOT, "include")]


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(ROOT, "include", "ssm_scan.h")])


def _deps(path: str, seen=None) -> set:
    """The file and every file it #includes with quotes, recursively (paths resolved relative to
    the including file)."""
    seen = set() if seen is None else seen
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    with open(path, encoding="utf-8") as fh:
        for line in fh:
            line = line.strip()
            if line.startswith("#include \""):
                inc = line.split('"')[1]
                _deps(os.path.join(os.path.dirname(path), inc), seen)
    return seen


def _obj(src: str) -> str:
    return os.path.join(BUILD_DIR, os.path.splitext(src)[0] + ".o")


def _obj_stale(src: str) -> bool:
    obj = _obj(src)
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in _deps(os.path.join(CSRC, src)))


def _compile(src: str, verbose: bool) -> str:
    obj = _obj(src)
    cmd = [NVCC, *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every kernel source for sm_100a and link the shared library; return its path.
    Objects are recompiled when they are older than any file they include; the library is
    relinked when an object was rebuilt or is newer than it."""
    os.makedirs(BUILD_DIR, exist_ok=True)
    todo = [s for s in SOURCES if force or _obj_stale(s)]  # objects older than their includes
    if todo:
        with cf.ThreadPoolExecutor(max_workers=len(todo)) as ex:
            list(ex.map(lambda s: _compile(s, verbose), todo))
    objs = [_obj(s) for s in SOURCES]
    if (not todo and os.path.exists(LIB)
            and all(os.path.getmtime(o) <= os.path.getmtime(LIB) for o in objs)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
