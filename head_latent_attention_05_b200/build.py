"""Compile libmla.so (all CUDA sources, one translation unit) for sm_100a, in-tree.

Also builds libmla_shortwait.so, the same sources with the attention kernel's pipeline waits
limited to 200 ns (its drains keep the long limit): the test build that makes a bounded wait
run out on purpose, so that the abort path (drain, MLA_ERR_DEVICE_TIMEOUT) can be tested
without faulting or hanging anything."""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "mla_abi.cu")
OUT = os.path.join(HERE, "libmla.so")
SHORTWAIT_OUT = os.path.join(HERE, "libmla_shortwait.so")
SHORTWAIT_NS = 200


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(out: str, defines, force: bool, verbose: bool) -> str:
    deps = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "mla.h"))
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(d) for d in deps)
        if os.path.getmtime(out) >= newest:
            return out
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xptxas", "-v" if verbose else "-O3"]
    cmd += [f"-D{d}" for d in defines]
    cmd += ["-o", out + ".tmp", SRC]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(out)}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(out + ".tmp", out)
    return out


def build_shortwait(force: bool = False) -> str:
    """The test build with 200 ns pipeline waits in the attention kernel."""
    return _compile(SHORTWAIT_OUT, [f"MLA_PIPE_WAIT_NS={SHORTWAIT_NS}ull"], force, False)


def build(force: bool = False, verbose: bool = False) -> str:
    out = _compile(OUT, [], force, verbose)
    build_shortwait(force)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(OUT)
