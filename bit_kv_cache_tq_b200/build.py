"""Build libtq.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m bit_kv_cache_tq_b200.build [--force]``.  The library is
rebuilt when any source under ``csrc/`` or ``include/`` is newer than it.
"""

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtq.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3",
    "-Xptxas", "-v",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale():
    if not os.path.exists(LIB):
        return True
    deps = sources() + _headers()
    built = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > built for p in deps)


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force=False, verbose=False):
    """Compile every CUDA/C++ source into libtq.so; return its path.  An object
    is recompiled when its source or any header is newer than it."""
    if not force and not _stale():
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    newest_header = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    objs, jobs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        if not force and os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_header):
            continue
        cmd = [nvcc(), "-c", src, "-o", obj, "-I", INCLUDE, "-I", CSRC] + NVCC_FLAGS
        jobs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)))
    failed = []
    for src, proc in jobs:  # the sources compile in parallel
        out, err = proc.communicate()
        if proc.returncode != 0:
            failed.append("nvcc failed for %s:\n%s\n%s" % (src, out, err))
        elif verbose:
            sys.stderr.write(err)
    if failed:
        raise RuntimeError("\n".join(failed))
    tmp = LIB + ".tmp"
    cmd = [nvcc(), "-shared", "-o", tmp] + objs + ["-gencode", "arch=compute_100a,code=sm_100a", "-lcudart_static",
                                                   "-ldl", "-lrt", "-lpthread"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (res.stdout, res.stderr))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
