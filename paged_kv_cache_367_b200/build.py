"""Build libpagedkv.so (sm_100a) in-tree with nvcc.

    python -m paged_kv_cache_367_b200.build [--force]

Each .cu (kernels) and .cpp (host runtime) under csrc/ is compiled by nvcc to an
object under _build/ and linked into paged_kv_cache_367_b200/libpagedkv.so.
nvcc cross-compiles, so no GPU is needed.
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import tempfile
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2",
         "--expt-relaxed-constexpr", "-I" + INCLUDE, "-I" + CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _deps_mtime():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return max(os.path.getmtime(f) for f in files)


def _compile(src, build_dir, extra):
    obj = os.path.join(build_dir, os.path.splitext(os.path.basename(src))[0] + ".o")
    subprocess.check_call([NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])
    return obj


def build(force: bool = False, extra_flags=(), out: str = LIB) -> str:
    """Compile csrc/*.cu and link `out`. `extra_flags` (e.g. -D tuning macros) go
    to every nvcc compile; such variants should be linked to a different path."""
    if not force and not extra_flags and os.path.exists(out) and \
            os.path.getmtime(out) >= _deps_mtime():
        return out
    if extra_flags:  # a variant: objects in a scratch folder, removed afterwards
        with tempfile.TemporaryDirectory(prefix="pkv_variant_") as d:
            return _build_into(d, list(extra_flags), out)
    os.makedirs(BUILD, exist_ok=True)
    return _build_into(BUILD, [], out)


def _build_into(build_dir: str, extra, out: str) -> str:
    srcs = sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, build_dir, extra), srcs))
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
