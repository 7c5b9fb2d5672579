"""Build the CPU oracle (test infrastructure) as oracle/liboracle.so, and
its mutation build (the same source with the planted mistakes compiled in,
-DQO_MUTATIONS) as oracle/liboracle_mut.so, which only the mutation test
loads.

The flags keep the arithmetic plain IEEE FP32: no contraction of a*b+c into a
fused operation (-ffp-contract=off), no fast-math reassociation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qstate_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
MUT_LIB = os.path.join(HERE, "liboracle_mut.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fno-finite-math-only", "-frounding-math", "-fopenmp", "-fPIC",
          "-shared", "-Wall", "-Wextra"]


def _compile(out: str, extra, force: bool) -> str:
    deps = [SRC, os.path.join(HERE, "qstate_oracle.h"), __file__]
    if not force and os.path.exists(out):
        if os.path.getmtime(out) >= max(os.path.getmtime(d) for d in deps):
            return out
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, *extra, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle and its mutation build if missing or older than
    their sources; returns the oracle's path."""
    _compile(MUT_LIB, ["-DQO_MUTATIONS"], force)
    return _compile(LIB, [], force)


def mutation_build(force: bool = False) -> str:
    return _compile(MUT_LIB, ["-DQO_MUTATIONS"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
