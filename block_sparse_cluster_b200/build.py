"""Build libda.so in-tree with nvcc for sm_100a (one nvcc per source file, in parallel).

    python block_sparse_cluster_b200/build.py [--force]

(Run it by path: importing the package loads libda.so, which this script produces.)
"""
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libda.so")
FAULT_LIB = os.path.join(HERE, "libda_fault.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-Xptxas", "-warn-spills", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps_mtime():
    files = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return max(os.path.getmtime(f) for f in files)


def _compile(src, extra=()):
    obj = os.path.join(BUILD, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    return src, obj, r.returncode, r.stdout + r.stderr


def _link(objs, lib):
    r = subprocess.run([NVCC, *ARCH, "-shared", "-o", lib, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc link of {os.path.basename(lib)} failed")


def build(verbose=False, force=False, extra=()):
    """Compile every csrc/*.cu for sm_100a and link libda.so, and the test build libda_fault.so
    (the same sources with DA_FAULT_INJECT defined: one withheld barrier arrival, for the test of
    the bounded device waits); skip what is up to date."""
    os.makedirs(BUILD, exist_ok=True)
    deps = _deps_mtime()
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < deps:
        srcs = sources()
        with cf.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda s: _compile(s, extra), srcs))
        failed = [r for r in results if r[2] != 0]
        for src, _, rc, log in results:
            if log.strip() and (verbose or rc != 0):
                sys.stderr.write(f"--- {os.path.basename(src)}\n{log}")
        if failed:
            raise RuntimeError("nvcc failed: " + ", ".join(os.path.basename(f[0]) for f in failed))
        _link([r[1] for r in results], LIB)
    if force or not os.path.exists(FAULT_LIB) or os.path.getmtime(FAULT_LIB) < deps:
        # only the attention kernel differs in the test build
        src = os.path.join(CSRC, "attention_tc.cu")
        obj = os.path.join(BUILD, "attention_tc_fault.o")
        r = subprocess.run([NVCC, *ARCH, *FLAGS, *extra, "-DDA_FAULT_INJECT", "-c", src, "-o", obj],
                           capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed: attention_tc.cu (fault-injection build)")
        objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + ".o") for s in sources()
                if os.path.basename(s) != "attention_tc.cu"]
        _link(objs + [obj], FAULT_LIB)
    return LIB


if __name__ == "__main__":
    t = build(verbose=True, force="--force" in sys.argv)
    print(t)
