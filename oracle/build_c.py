"""Build the oracle's plain-C helpers (test infrastructure only) with gcc.

  python -m oracle.build_c

The library goes next to its source (oracle/c/liboracle_c.so).  It is
compiled without floating-point contraction or fast-math, so each operation
rounds as the numpy oracle's does.
"""

from __future__ import annotations

import pathlib
import shutil
import subprocess

HERE = pathlib.Path(__file__).resolve().parent / "c"
SRC = sorted(HERE.glob("*.c"))
LIB = HERE / "liboracle_c.so"
FLAGS = ["-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
         "-fno-fast-math", "-fno-unsafe-math-optimizations"]


def build(force: bool = False) -> pathlib.Path:
    if not force and LIB.exists() and all(s.stat().st_mtime <= LIB.stat().st_mtime for s in SRC):
        return LIB
    cc = shutil.which("gcc") or shutil.which("cc")
    if not cc:
        raise RuntimeError("gcc not found: the oracle's C helpers need a C compiler")
    tmp = LIB.with_suffix(".so.tmp")
    r = subprocess.run([cc, *FLAGS, "-o", str(tmp), *map(str, SRC), "-lm"], capture_output=True,
                       text=True)
    if r.returncode != 0:
        raise RuntimeError(f"gcc failed:\n{r.stdout}\n{r.stderr}")
    tmp.replace(LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
