"""Build the C-ABI library ``libsconvkv.so`` (sm_100a) in-tree with nvcc.

The host code (``csrc/sconv_kv.cu``) and the kernel-instance translation
units (``csrc/inst_*.cu``) are compiled to objects in parallel, then linked
into one shared library.
"""
import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsconvkv.so")
SOURCES = [os.path.join(CSRC, "sconv_kv.cu")] + sorted(
    os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.startswith("inst_") and f.endswith(".cu"))
DEPS = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xptxas", "-v",
                        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def needs_build(out=LIB):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in DEPS if os.path.exists(d))


def _compile(src, obj, extra):
    cmd = [nvcc(), *COMPILE_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    return res.stdout + res.stderr


def build(out=LIB, quiet=True, extra=()):
    """Compile every translation unit (in parallel) and link `out`."""
    objdir = os.path.join(ROOT, "_build", os.path.basename(out) + ".objs")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, os.path.basename(s)[:-3] + ".o") for s in SOURCES]
    workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        logs = list(ex.map(lambda so: _compile(so[0], so[1], extra), zip(SOURCES, objs)))
    cmd = [nvcc(), *ARCH, "-shared", "-o", out, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    with open(out + ".ptxas.txt", "w") as f:
        f.write("".join(logs) + res.stdout + res.stderr)
    if not quiet:
        sys.stderr.write("".join(logs))
    return out


if __name__ == "__main__":
    print(build(quiet=False))
