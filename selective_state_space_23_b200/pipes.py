"""Per-SM, per-clock throughput of the pipes the scan kernels use (FP32 FMA scalar and packed,
MUFU ex2), measured on the current GPU: the unit rates behind the forward kernel's arithmetic
roofline.  ``python -m selective_state_space_23_b200.pipes`` builds the probe (its own small
library, not part of the scan library) and prints one JSON line: per pipe, operations per SM
per clock64 tick and per nanosecond, and the clock64 rate in MHz that links the two.
"""
import ctypes
import json
import os
import subprocess
import sys

from .build import ARCH, CSRC, NVCC, PKG

LIB = os.path.join(PKG, "libssm_pipes.so")
SRC = os.path.join(CSRC, "pipe_rates.cu")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = [NVCC, *ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-o", LIB, SRC,
               "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for pipe_rates.cu:\n{r.stdout}\n{r.stderr}")
    return LIB


def measure(iters: int = 4096, ctas_per_sm: int = 4, threads: int = 256) -> dict:
    lib = ctypes.CDLL(build())
    f = lib.ssm_pipe_probe
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.POINTER(ctypes.c_double)]
    out = {"ctas_per_sm": ctas_per_sm, "threads_per_cta": threads, "iters": iters}
    for kind, name in ((0, "ffma_fp32_ops"), (1, "ffma2_fp32_ops"), (2, "mufu_ex2")):
        rate = (ctypes.c_double * 3)()
        rc = f(kind, iters, ctas_per_sm, threads, rate)
        if rc != 0:
            raise RuntimeError(f"pipe probe {name} failed ({rc})")
        out[name + "_per_clk_per_sm"] = rate[0]
        out[name + "_per_ns_per_sm"] = rate[1]
        out[name + "_sm_mhz"] = rate[2]
    return out


if __name__ == "__main__":
    print(json.dumps(measure()))
    sys.exit(0)
