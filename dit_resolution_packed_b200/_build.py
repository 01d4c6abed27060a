"""Builds ``libpackattn.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

The library links the CUDA runtime statically, so it loads on a machine without
a GPU (only calls that reach the device need one).
"""
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpackattn.so")
SOURCES = ["packattn.cu"]
HEADERS = ["sm100_ptx.cuh", "schedule.cuh", "attn_fwd_sm100.cuh", "attn_fwd_fp8_sm100.cuh", "attn_bwd_sm100.cuh",
           "gemm_sm100.cuh", "exp2_poly.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "packattn.h"))
    files.append(os.path.abspath(__file__))
    return files


def nvcc_command(out=LIB, extra=()):
    return [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
            "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "-cudart", "static",
            "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic",
            "-I", os.path.join(ROOT, "include"), "-I", CSRC,
            *extra, "-o", out] + [os.path.join(CSRC, f) for f in SOURCES]


# The forward kernels split their register pool with setmaxnreg; the split is
# only valid if they are compiled at exactly this count.  The backward kernel runs
# 16 warps at 128 registers each (the whole register file) without a split.
LAUNCH_REGS = 168
BWD_MAX_REGS = 128


def _check_registers(ptxas_log):
    """Fails the build unless each forward attention kernel uses exactly LAUNCH_REGS
    registers and the backward kernel at most BWD_MAX_REGS."""
    kernel = None
    seen = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            kernel = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and kernel and any(n in kernel for n in ("attn_fwd_kernel", "attn_fwd_fp8_kernel", "attn_bwd_kernel")):
            regs = int(m.group(1))
            if "attn_bwd_kernel" in kernel:
                if regs > BWD_MAX_REGS:
                    raise RuntimeError(f"{kernel}: {regs} registers, at most {BWD_MAX_REGS} for 16 warps")
            elif regs != LAUNCH_REGS:
                raise RuntimeError(f"{kernel}: {regs} registers, expected {LAUNCH_REGS} for the register split")
            seen += 1
    if seen == 0:
        raise RuntimeError("no attention kernel in the ptxas report")
    return seen


def build(force=False, verbose=False, ptxas_info=False):
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in _inputs())
        if os.path.getmtime(LIB) >= newest:
            return LIB
    tmp = LIB + ".tmp"
    cmd = nvcc_command(tmp, ["-Xptxas", "-v"])
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed")
    if ptxas_info:
        sys.stderr.write(res.stderr)
    _check_registers(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True, ptxas_info="-v" in sys.argv))
