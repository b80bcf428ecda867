"""Build the oracle's shared library with the host C compiler.

Test infrastructure only: the oracle is compiled with strict IEEE semantics
(no fast-math, no FMA contraction) so that its double-precision sums are the
plain left-to-right sums the source spells out.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sconv_kv_oracle.c")
LIB = os.path.join(HERE, "liboracle_sconv_kv.so")

CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(src=SRC, out=LIB, extra=(), quiet=True):
    """Compile `src` into the shared library `out`; return `out`."""
    cc = os.environ.get("CC", "gcc")
    cmd = [cc, *CFLAGS, *extra, "-o", out, src, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + " ".join(cmd) + "\n" +
                           res.stdout + res.stderr)
    if not quiet and res.stderr:
        sys.stderr.write(res.stderr)
    return out


def needs_build(out=LIB, src=SRC):
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build(quiet=False))
