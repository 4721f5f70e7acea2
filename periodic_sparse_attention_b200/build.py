"""Build the CUDA library libpiattn.so in-tree (nvcc, sm_100a only).

    python -m periodic_sparse_attention_b200.build [--force]

The library is one translation unit (csrc/pi_attn.cu including the kernel headers) compiled for
sm_100a with -lineinfo; it exports the C ABI declared in include/pi_attn.h.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libpiattn.so")
MAIN = os.path.join(HERE, "csrc", "pi_attn.cu")
_lock = threading.Lock()


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def command(out: str, extra=()):
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC,-O2", "-shared", *extra, MAIN, "-o", out]


def stale() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    with _lock:
        if force or stale():
            tmp = SO + f".tmp{os.getpid()}"
            cmd = command(tmp, ["-Xptxas", "-v"] if verbose else [])
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
            if verbose:
                sys.stderr.write(r.stderr)
            os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
