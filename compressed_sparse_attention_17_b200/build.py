"""Build libcsa.so (the CUDA kernels and the C ABI) in-tree for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
LIB = PKG / "libcsa.so"
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr", "-Xptxas", "-v",
]


def sources():
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) + \
        [PKG.parent / "include" / "csa.h"]


def _compile(src: Path, obj: Path):
    cmd = [NVCC, *NVCC_FLAGS, "-c", str(src), "-o", str(obj)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    return src, cmd, res


def build(force: bool = False, verbose: bool = False) -> Path:
    """Compile every csrc/*.cu for sm_100a (in parallel) and link libcsa.so."""
    newest = max(p.stat().st_mtime for p in sources())
    if not force and LIB.exists() and LIB.stat().st_mtime >= newest:
        return LIB
    objdir = PKG / "_build"
    objdir.mkdir(exist_ok=True)
    units = sorted(CSRC.glob("*.cu"))
    headers = [p for p in sources() if p.suffix in (".cuh", ".h")]
    newest_header = max(p.stat().st_mtime for p in headers)

    def stale(u: Path) -> bool:
        o = objdir / (u.stem + ".o")
        return force or not o.exists() or o.stat().st_mtime < max(u.stat().st_mtime, newest_header)

    todo = [u for u in units if stale(u)]
    log = []
    with ThreadPoolExecutor(max_workers=max(1, min(8, len(todo)))) as ex:
        results = list(ex.map(lambda u: _compile(u, objdir / (u.stem + ".o")), todo))
    failed = False
    for src, cmd, res in results:
        log.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        if res.returncode != 0:
            failed = True
            sys.stderr.write(res.stdout + res.stderr)
    (objdir / "build.log").write_text("\n".join(log))
    if failed:
        raise RuntimeError("nvcc failed building libcsa.so (see _build/build.log)")
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           *[str(objdir / (u.stem + ".o")) for u in units], "-o", str(tmp)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libcsa.so")
    if verbose:
        sys.stdout.write("\n".join(log))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
