"""Build the in-tree CUDA library libmx.so for sm_100a (nvcc, no JIT cache).

Every csrc/*.cu file is compiled to its own object (in parallel, one nvcc per file,
under _build/), then the objects are linked into libmx.so.  An object is rebuilt
when its source, a csrc header or an include/ header is newer than it.
"""
from __future__ import annotations

import glob
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmx.so")
OBJ_DIR = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-v",
          "--expt-relaxed-constexpr"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def _headers() -> list[str]:
    return glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _obj(src: str) -> str:
    return os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str) -> tuple[str, subprocess.CompletedProcess]:
    out = _obj(src)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [NVCC, *CFLAGS, "-I", os.path.join(ROOT, "include"), "-c", "-o", tmp, src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode == 0:
        os.replace(tmp, out)
    return " ".join(cmd), res


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ and link libmx.so (static cudart); return its path."""
    os.makedirs(OBJ_DIR, exist_ok=True)
    hdrs = _headers()
    todo = [s for s in sources() if force or _stale(_obj(s), [s, *hdrs])]
    logs = []
    failed = None
    if todo:
        with ThreadPoolExecutor(max(1, min(len(todo), os.cpu_count() or 4))) as pool:
            for cmd, res in pool.map(_compile, todo):
                logs.append(cmd + "\n" + res.stdout + res.stderr)
                if res.returncode != 0 and failed is None:
                    failed = res.stderr
    objs = [_obj(s) for s in sources()]
    if failed is None and (todo or _stale(LIB, objs)):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        logs.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        if res.returncode != 0:
            failed = res.stderr
        else:
            os.replace(tmp, LIB)
    if logs:
        with open(os.path.join(HERE, "build.log"), "w") as f:
            f.write("\n".join(logs))
    if failed is not None:
        raise RuntimeError(f"nvcc failed (see {os.path.join(HERE, 'build.log')}):\n{failed[-4000:]}")
    if verbose:
        print("\n".join(logs))
    return LIB


if __name__ == "__main__":
    print(build(force=True))
