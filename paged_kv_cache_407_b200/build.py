"""Build libpkv.so (the C-ABI CUDA library) in-tree for B200 (sm_100a).

Usage: ``python -m paged_kv_cache_407_b200.build [-v] [--check]``.  Compiles
every ``csrc/*.cu`` with nvcc and every host-only ``csrc/*.cpp`` with the host
compiler into ``_build/`` and links ``paged_kv_cache_407_b200/libpkv.so``
(CUDA runtime linked statically).  ``--check`` also links the check build
``libpkv_check.so``: the sources that test ``PKV_CHECK`` compiled again with it
defined (into ``_build/check/``), the other objects shared with libpkv.so.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG_DIR, "_build")
LIB_PATH = os.path.join(PKG_DIR, "libpkv.so")
CHECK_LIB_PATH = os.path.join(PKG_DIR, "libpkv_check.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC,
]


CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-fvisibility=hidden", "-Wall", "-Wextra", "-I", INCLUDE, "-I", CSRC]


def cxx_path() -> str:
    cand = os.environ.get("CXX") or shutil.which("g++") or shutil.which("c++")
    if not cand:
        raise RuntimeError("no host C++ compiler found to build libpkv")
    return cand


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libpkv")
    return cand


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def check_sources() -> list[str]:
    """The sources whose code depends on PKV_CHECK."""
    out = []
    for src in sources():
        with open(src, encoding="utf-8") as f:
            if "PKV_CHECK" in f.read():
                out.append(src)
    return out


def _object(src: str, out_dir: str) -> str:
    return os.path.join(out_dir, os.path.splitext(os.path.basename(src))[0] + ".o")


def _compile(src: str, verbose: bool, ptxas_info: bool, out_dir: str | None = None, check: bool = False) -> str:
    obj = _object(src, out_dir or BUILD_DIR)
    defs = ["-DPKV_CHECK=1"] if check else []
    if src.endswith(".cpp"):
        cmd = [cxx_path(), *CXX_FLAGS, *defs, "-c", src, "-o", obj]
    else:
        cmd = [nvcc_path(), *ARCH_FLAGS, *NVCC_FLAGS, *defs, "-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"compiling {src} failed:\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        sys.stderr.write(res.stdout + res.stderr)
    return obj


def _stale(objs_srcs, lib_path: str | None = None) -> bool:
    lib_path = lib_path or LIB_PATH
    if not os.path.exists(lib_path):
        return True
    lib_t = os.path.getmtime(lib_path)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    newest = max(os.path.getmtime(p) for p in [*objs_srcs, *headers, __file__])
    return newest > lib_t


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    srcs = sources()
    if not force and not ptxas_info and not _stale(srcs):
        return LIB_PATH
    os.makedirs(BUILD_DIR, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, ptxas_info), srcs))
    _link(objs, LIB_PATH)
    return LIB_PATH


def _link(objs, lib_path: str) -> None:
    tmp = lib_path + ".tmp"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib_path)


def build_check(verbose: bool = False, force: bool = False) -> str:
    """libpkv_check.so: libpkv.so's objects, except that the sources which
    test PKV_CHECK are compiled again with it defined."""
    srcs = sources()
    if not force and not _stale(srcs, CHECK_LIB_PATH):
        return CHECK_LIB_PATH
    build(verbose=verbose)
    check_dir = os.path.join(BUILD_DIR, "check")
    os.makedirs(check_dir, exist_ok=True)
    checked = check_sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs_c = list(ex.map(lambda s: _compile(s, verbose, False, check_dir, check=True), checked))
    objs = []
    for src in srcs:
        if src in checked:
            objs.append(objs_c[checked.index(src)])
        else:
            obj = _object(src, BUILD_DIR)
            objs.append(obj if os.path.exists(obj) else _compile(src, verbose, False))
    _link(objs, CHECK_LIB_PATH)
    return CHECK_LIB_PATH


if __name__ == "__main__":
    v = "-v" in sys.argv
    print(build(verbose=v, force=True, ptxas_info=v))
    if "--check" in sys.argv:
        print(build_check(verbose=v, force=True))
