"""Build the sm_100a shared library ``libmla_b200.so`` in-tree.

Every ``csrc/*.cu`` file is compiled by nvcc for ``sm_100a`` only and linked
into one shared library with the CUDA runtime linked statically; the driver
entry point for tensor-map encoding is fetched at run time, so the library
loads on a machine without a GPU driver (symbols can be listed there).

    python -m latent_attention_b200.build [--force] [-j N] [--verbose]
"""
import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmla_b200.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc",
                 shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _compile(src, obj, extra, verbose):
    cmd = [nvcc(), "-c", src, "-o", obj] + NVCC_FLAGS + extra
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build(force=False, jobs=None, verbose=False, ptxas_info=False):
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = _deps()
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    todo = []
    objs = []
    for s in sources:
        o = os.path.join(BUILD, os.path.basename(s) + ".o")
        objs.append(o)
        if force or ptxas_info or _stale(o, [s] + deps):
            todo.append((s, o))
    logs = {}
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or os.cpu_count()) as ex:
            futs = {ex.submit(_compile, s, o, extra, verbose): s for s, o in todo}
            for f in cf.as_completed(futs):
                logs[futs[f]] = f.result()
    if todo or _stale(LIB, objs):
        cmd = [nvcc(), "-shared", "-o", LIB] + ARCH + objs + ["-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB, logs


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-j", type=int, default=None)
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true",
                    help="rebuild with -Xptxas -v and print register/smem use")
    a = ap.parse_args(argv)
    lib, logs = build(a.force, a.j, a.verbose, a.ptxas_info)
    if a.ptxas_info:
        for s, log in sorted(logs.items()):
            print(f"== {os.path.basename(s)}\n{log}")
    print(lib)


if __name__ == "__main__":
    sys.exit(main())
