"""Build step: compile the CUDA sources into the in-tree C-ABI library.

    python -m sparse_transformer_attention_b200.build [--force] [--debug]

nvcc cross-compiles for sm_100a (B200); no GPU is needed to build.  Each
translation unit is compiled to an object in parallel (relocatable device
code is not needed: no kernel calls across files), then linked into
`libcondensate_attn.so`.  `--debug` compiles the same sources with CA_DEBUG
into `libcondensate_attn_debug.so` (kernels that also check the indexes the
release build keeps in range by construction, reporting CA_ERR_BOUNDS).
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libcondensate_attn.so")
OBJ_DIR = os.path.join(HERE, "_build")
LIB_DEBUG = os.path.join(HERE, "libcondensate_attn_debug.so")
OBJ_DIR_DEBUG = os.path.join(HERE, "_build_debug")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"),
                 "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _obj(src: str, obj_dir: str = OBJ_DIR) -> str:
    return os.path.join(obj_dir, os.path.basename(src) + ".o")


def _stale(target: str, inputs: list) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in inputs)


def build(force: bool = False, verbose: bool = False,
          debug: bool = False) -> str:
    """Compile (incrementally) and link the release library, or with
    debug=True the CA_DEBUG one; returns the library's path."""
    obj_dir, lib = (OBJ_DIR_DEBUG, LIB_DEBUG) if debug else (OBJ_DIR, LIB)
    flags = NVCC_FLAGS + (["-DCA_DEBUG"] if debug else [])
    os.makedirs(obj_dir, exist_ok=True)
    nvcc = _nvcc()
    deps = _deps()
    todo = [s for s in sources()
            if force or _stale(_obj(s, obj_dir), [s] + deps)]

    def compile_one(src):
        cmd = [nvcc, *flags, "-I", INCLUDE, "-c", "-o", _obj(src, obj_dir),
               src]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)

    with concurrent.futures.ThreadPoolExecutor(max_workers=8) as ex:
        list(ex.map(compile_one, todo))
    objs = [_obj(s, obj_dir) for s in sources()]
    if force or todo or _stale(lib, objs):
        cmd = [nvcc, *ARCH, "-shared", "-o", lib + ".tmp", *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                debug="--debug" in sys.argv))
