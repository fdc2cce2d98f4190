"""Build libnvfp4.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m scale_calibration_nvfp4_b200.build [--force] [--verbose]

Each ``csrc/*.cu`` file is compiled by nvcc for ``arch=compute_100a,
code=sm_100a`` and linked into ``scale_calibration_nvfp4_b200/libnvfp4.so``
with the static CUDA runtime.  Objects are rebuilt only when their source, a
shared header or this script is newer; the library is relinked when an object
is.  Sources that instantiate CUTLASS/CuTe templates (the FP4 GEMM) get the
header tree vendored in the environment's site-packages.
"""
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libnvfp4.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "-I" + os.path.join(ROOT, "include")]


def _nvcc():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libnvfp4.so")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    files = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    files.append(os.path.abspath(__file__))
    return files


def _shared_inputs():
    files = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    files.append(os.path.abspath(__file__))
    return files


# The CUTLASS release the two template sources (gemm_fp4.cu, gram_full.cu) were
# written and tested against; the header tree is taken from the environment,
# so its version is checked rather than assumed.
CUTLASS_VERSION = (4, 5, 0)


def cutlass_version(include_dir):
    """(major, minor, patch) from cutlass/version.h under include_dir."""
    v = {}
    with open(os.path.join(include_dir, "cutlass", "version.h")) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == "#define" and parts[1] in (
                    "CUTLASS_MAJOR", "CUTLASS_MINOR", "CUTLASS_PATCH"):
                v[parts[1]] = int(parts[2])
    return v.get("CUTLASS_MAJOR"), v.get("CUTLASS_MINOR"), v.get("CUTLASS_PATCH")


def cutlass_include():
    """CUTLASS/CuTe headers vendored with flashinfer (header-only use), of
    the release CUTLASS_VERSION names."""
    import importlib.util
    spec = importlib.util.find_spec("flashinfer")
    for base in (spec.submodule_search_locations or []) if spec else []:
        inc = os.path.join(base, "data", "cutlass", "include")
        util = os.path.join(base, "data", "cutlass", "tools", "util", "include")
        if os.path.isdir(os.path.join(inc, "cute")):
            found = cutlass_version(inc)
            if found != CUTLASS_VERSION:
                raise RuntimeError("CUTLASS headers at %s are version %s; this library's "
                                   "template sources need %s" % (inc, found, CUTLASS_VERSION))
            return [inc, util]
    raise RuntimeError("CUTLASS/CuTe headers not found (expected under flashinfer/data/cutlass)")


def _uses_cutlass(src):
    with open(src) as f:
        return "#include <cute/" in f.read()


def _obj(src):
    return os.path.join(BUILD_DIR, os.path.basename(src) + ".o")


def _stale(src, obj):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(f) > t for f in [src] + _shared_inputs())


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs()) and \
        all(os.path.exists(_obj(s)) and os.path.getmtime(_obj(s)) <= t for s in sources())


def build(force=False, verbose=False, ptxas_info=False):
    if not force and up_to_date():
        return LIB
    nvcc = _nvcc()
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    for src in sources():
        obj = _obj(src)
        objs.append(obj)
        if not (force or ptxas_info or _stale(src, obj)):
            continue
        cmd = [nvcc] + ARCH + NVCC_FLAGS
        if _uses_cutlass(src):
            cmd += ["--expt-relaxed-constexpr", "-Xcompiler", "-Wno-unused-parameter",
                    "-diag-suppress", "20012"]
            cmd += ["-I" + d for d in cutlass_include()]
        cmd += ["-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [nvcc] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                ptxas_info="--ptxas" in sys.argv))
