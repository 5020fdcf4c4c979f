"""Build libdfk.so (the sm_100a kernels and the C ABI) in-tree with nvcc.

    python -m swiglu_mlp_dfk_b200.build [--force] [-j N]

Every CUDA source is compiled with
``-gencode arch=compute_100a,code=sm_100a -lineinfo -O3`` (no fast-math:
SiLU uses the accurate expf and IEEE division), objects go to ``_build/`` and
the shared library to ``swiglu_mlp_dfk_b200/libdfk.so``.  The CUDA runtime is
linked statically and only the ``dfk_*`` C symbols are exported, so the
library loads with or without PyTorch in the process.

A second, checked build (``-DDFK_CHECKED``: every global store of a result
and the activation loads test their index against the tensor's extent and
record the first failure in the device status word instead of accessing
memory) goes to ``_build/checked/`` and ``swiglu_mlp_dfk_b200/libdfk_checked.so``;
the binding loads it when ``DFK_CHECKED=1`` is set.
"""
import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdfk.so")
LIB_CHECKED = os.path.join(PKG, "libdfk_checked.so")

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                 "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hs + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def _compile(src, force, hdr_time, outdir, extra):
    obj = os.path.join(outdir, os.path.basename(src)[:-3] + ".o")
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= max(
            os.path.getmtime(src), hdr_time):
        return obj, None
    cmd = [NVCC] + CFLAGS + extra + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        return obj, "%s\n%s%s" % (" ".join(cmd), r.stdout, r.stderr)
    return obj, None


def _build_one(lib, outdir, extra, force, jobs, verbose):
    os.makedirs(outdir, exist_ok=True)
    srcs = sources()
    hdr_time = _newest(headers())
    if (not force and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(_newest(srcs), hdr_time)):
        return lib
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    objs, errors = [], []
    with cf.ThreadPoolExecutor(max_workers=jobs) as ex:
        for obj, err in ex.map(lambda s: _compile(s, force, hdr_time, outdir, extra), srcs):
            objs.append(obj)
            if err:
                errors.append(err)
    if errors:
        raise RuntimeError("nvcc failed:\n" + "\n".join(errors))
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [NVCC] + ARCH + ["-shared", "-Xcompiler", "-fvisibility=hidden", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s%s" % (" ".join(cmd), r.stdout, r.stderr))
    os.replace(tmp, lib)
    if verbose:
        print(lib)
    return lib


def build(force: bool = False, jobs: int = 0, verbose: bool = False,
          checked: bool = True) -> str:
    """Compile every .cu under csrc/ and link libdfk.so (and, with `checked`,
    the bounds-checked libdfk_checked.so); returns the path of libdfk.so."""
    lib = _build_one(LIB, BUILD, [], force, jobs, verbose)
    if checked:
        _build_one(LIB_CHECKED, os.path.join(BUILD, "checked"), ["-DDFK_CHECKED"], force, jobs,
                   verbose)
    return lib


if __name__ == "__main__":
    j = 0
    if "-j" in sys.argv:
        j = int(sys.argv[sys.argv.index("-j") + 1])
    build(force="--force" in sys.argv, jobs=j, verbose=True)
