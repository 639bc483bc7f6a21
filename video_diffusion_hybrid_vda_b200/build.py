"""Build libvdn.so in-tree from csrc/*.cu for sm_100a (nvcc cross-compiles
without a GPU).  Usage: ``python -m video_diffusion_hybrid_vda_b200.build``
(``--force`` rebuilds, ``-v`` prints ptxas register and spill counts,
``--debug-bounds`` builds the bounds-checking libvdn_debug.so instead).

Build-time switches of the kernels are passed as preprocessor definitions
in ``VDN_NVCC_DEFINES`` (comma-separated ``NAME=VALUE``), e.g.
``VDN_NVCC_DEFINES=VDN_EXP2_FMA_PAIRS=4`` for the window Softmax's
FMA-pipe share of the exponentials; a build with definitions should be
forced, since the up-to-date check looks at file times only."""

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libvdn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden"]


def nvcc():
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; libvdn needs the CUDA toolkit to build")
    return path


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) +
                  glob.glob(os.path.join(os.path.dirname(HERE), "include", "*.h")))


DEBUG_LIB = os.path.join(HERE, "libvdn_debug.so")  # VDN_DEBUG_BOUNDS=1 variant


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in sources() + headers() + [__file__])


def defines():
    """-D flags from VDN_NVCC_DEFINES (comma-separated NAME=VALUE)."""
    spec = os.environ.get("VDN_NVCC_DEFINES", "").strip()
    out = []
    for item in filter(None, (x.strip() for x in spec.split(","))):
        name = item.split("=", 1)[0]
        if not name.isidentifier():
            raise ValueError(f"VDN_NVCC_DEFINES: bad definition {item!r}")
        out.append("-D" + item)
    return out


def build(force=False, verbose=False, jobs=None, debug_bounds=False):
    """Compile every csrc/*.cu to an object and link libvdn.so, or with
    ``debug_bounds`` the libvdn_debug.so variant built with
    VDN_DEBUG_BOUNDS=1 (every hand-computed global store checked against
    its tensor's extents on the device)."""
    lib = DEBUG_LIB if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    objdir = os.path.join(HERE, "_build_debug" if debug_bounds else "_build")
    os.makedirs(objdir, exist_ok=True)
    inc = ["-I", os.path.join(os.path.dirname(HERE), "include"), *defines()]
    if debug_bounds:
        inc.append("-DVDN_DEBUG_BOUNDS=1")
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        objs.append(obj)
        cmd = [nvcc(), *ARCH, *FLAGS, *inc, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    failed = []
    for src, p in procs:
        out = p.communicate()[0].decode()
        if verbose or p.returncode:
            sys.stdout.write(out)
        if p.returncode:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed on: " + ", ".join(failed))
    tmp = lib + ".tmp"
    subprocess.check_call([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-ldl"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
