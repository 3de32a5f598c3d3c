"""Build the CPU oracle shared library (test infrastructure only).

    python oracle/build.py        # writes oracle/liboref.so

Plain C11, -O2 without fast-math and with fp contraction off, so that every
fp64 operation in the oracle is one correctly rounded IEEE operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["oref_fp.c", "oref_format_a.c", "oref_format_b.c"]
LIB = os.path.join(HERE, "liboref.so")


def build(out: str = LIB, extra_flags=(), src_dir: str = HERE) -> str:
    srcs = [os.path.join(src_dir, s) for s in SOURCES]
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-Werror", *extra_flags,
           "-I", src_dir, *srcs, "-lm", "-o", out]
    subprocess.run(cmd, check=True)
    return out


def needs_build(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = SOURCES + ["oref.h", "build.py"]
    return any(os.path.getmtime(os.path.join(HERE, d)) > t for d in deps)


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
