"""Build libstreamkl.so in-tree with nvcc for sm_100a (cross-compiles without a GPU)."""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys
import tempfile
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
INCLUDE = ROOT / "include"
LIB = PKG / "libstreamkl.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-shared", "-cudart", "shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu"))


def _stale(out: Path) -> bool:
    if not out.exists():
        return True
    t = out.stat().st_mtime
    deps = list(CSRC.glob("*.cu")) + list(CSRC.glob("*.cuh")) + list(CSRC.glob("*.h")) + \
        list(INCLUDE.glob("*.h")) + [Path(__file__)]
    return any(p.stat().st_mtime > t for p in deps)


def build(force: bool = False, extra: list[str] | None = None, out: Path = LIB) -> Path:
    """Compile every source to an object in parallel, then link the shared library."""
    if not force and not extra and not _stale(out):
        return out
    tmp = out.with_name(out.name + f".tmp{os.getpid()}")
    flags = [*NVCC_FLAGS, *(extra or []), f"-I{INCLUDE}", f"-I{CSRC}"]
    compile_flags = [f for f in flags if f not in ("-shared", "-cudart", "shared")]
    with tempfile.TemporaryDirectory(prefix="streamkl_build_") as objdir:
        objs = [Path(objdir) / (src.stem + ".o") for src in sources()]
        jobs = [[nvcc(), *compile_flags, "-c", str(src), "-o", str(obj)]
                for src, obj in zip(sources(), objs)]
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as pool:
            for res in pool.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs):
                sys.stderr.write(res.stdout + res.stderr)
                if res.returncode != 0:
                    raise subprocess.CalledProcessError(res.returncode, res.args)
        subprocess.run([nvcc(), *flags, *map(str, objs), "-o", str(tmp)], check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, extra=[a for a in sys.argv[1:] if a != "--force"]))
