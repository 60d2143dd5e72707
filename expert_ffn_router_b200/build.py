"""Build libmoe.so (sm_100a) in-tree, and its bounds-checked twin.

    python expert_ffn_router_b200/build.py [--force] [--verbose]

(run it by path: importing the package loads the library this script builds)

Each .cu translation unit under csrc/ is compiled in parallel with
``nvcc -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and the objects
are linked into expert_ffn_router_b200/libmoe.so (static CUDA runtime, no
torch dependency).  libmoe_bounds.so is the same library compiled with
MOE_BOUNDS: every index the kernels read from data is range-checked and a
violation is recorded as MOE_EDEVICE in the workspace's status word (the
package loads it instead when MOE_LIBRARY=bounds).  A build is skipped when
its library is newer than every source and header.
"""
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")
LIB_BOUNDS = os.path.join(PKG, "libmoe_bounds.so")
BUILD = os.path.join(PKG, "_build")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments, whitespace runs collapsed; string
    and character literals are kept as written."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_hash() -> str:
    """Hash of the code (comments and layout ignored) of every source and
    header the library is built from: ties a recorded ncu traffic figure to
    the kernel it was measured on."""
    import hashlib
    h = hashlib.sha256()
    for p in sorted(_deps()):
        if p.endswith(".py"):
            continue
        with open(p, encoding="utf-8") as fh:
            h.update(os.path.basename(p).encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, verbose: bool, extra, tag: str) -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + tag + ".o")
    cmd = [nvcc()] + NVCC_FLAGS + list(extra) + (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def _build_one(lib: str, extra, tag: str, force: bool, verbose: bool) -> str:
    if not force and up_to_date(lib):
        return lib
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, tag), sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp] + objs + ["-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, bounds: bool = True) -> str:
    """Build libmoe.so (and libmoe_bounds.so unless bounds=False); returns libmoe.so's path."""
    _build_one(LIB, [], "", force, verbose)
    if bounds:
        _build_one(LIB_BOUNDS, ["-DMOE_BOUNDS"], ".bounds", force, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
