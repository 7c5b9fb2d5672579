"""Build the CUDA library libqstate.so in-tree for B200 (sm_100a).

Every translation unit under csrc/ is compiled by nvcc for
compute_100a/sm_100a with -fmad=false (no implicit contraction of a*b+c;
the kernels use explicit rounding intrinsics anyway) and linked with the
static CUDA runtime into ssm_decode_step_b200/libqstate.so.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build", "qstate")
LIB = os.path.join(HERE, "libqstate.so")
HEADER = os.path.join(ROOT, "include", "qstate.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVFLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC",
                  "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]
# Extra nvcc flags (e.g. -DQS_MIN_BLOCKS=3) for tuning builds.
NVFLAGS += os.environ.get("QSTATE_NVCC_FLAGS", "").split()


def flags_key() -> str:
    """The nvcc flags without include directories (which name this checkout's
    location): what the library's code depends on."""
    out, skip = [], False
    for f in NVFLAGS:
        if skip:
            skip = False
        elif f == "-I":
            skip = True
        elif not f.startswith("-I"):
            out.append(f)
    return " ".join(out)


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    return [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [HEADER, __file__]


STAMP = LIB + ".flags"
# ptxas's resource report (registers, spills, shared memory per kernel) of the last build
PTXAS_LOG = os.path.join(BUILD, "ptxas.log")


def _up_to_date() -> bool:
    """The library exists, is newer than every source, and was built with
    the same nvcc flags."""
    if not (os.path.exists(LIB) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        if f.read() != flags_key():
            return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and _up_to_date():
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    cc = nvcc()
    # the resource report changes no code; it is kept in PTXAS_LOG
    extra = ["-Xptxas", "-v"]

    def compile_one(src):
        obj = os.path.join(BUILD, os.path.basename(src) + ".o")
        cmd = [cc, *NVFLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        return obj, r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, _sources()))
    with open(PTXAS_LOG, "w") as f:
        for _, log in results:
            f.write(log)
    if verbose or ptxas_info:
        for _, log in results:
            if log:
                sys.stderr.write(log)
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *[o for o, _ in results]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(flags_key())
    return LIB


def ptxas_report() -> dict:
    """{kernel (mangled name): {"registers": n, "spill_stores": bytes,
    "spill_loads": bytes}} from the last build's ptxas report (rebuilt when
    the report is missing)."""
    import re
    if not os.path.exists(PTXAS_LOG):
        build(force=True)
    out, cur = {}, None
    with open(PTXAS_LOG) as f:
        for line in f:
            m = re.search(r"Compiling entry function '(\S+)'", line)
            if m:
                cur = m.group(1)
                out[cur] = {}
                continue
            m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
            if m and cur:
                out[cur]["spill_stores"] = int(m.group(1))
                out[cur]["spill_loads"] = int(m.group(2))
            m = re.search(r"Used (\d+) registers", line)
            if m and cur:
                out[cur]["registers"] = int(m.group(1))
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                ptxas_info="--ptxas" in sys.argv))
