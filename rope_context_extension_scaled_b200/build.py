"""Build librcx.so in-tree for sm_100a.

    python -m rope_context_extension_scaled_b200.build [--force] [-v]

Each csrc/*.cu file is one translation unit (the C-ABI host code, and one
unit per kernel family); they are compiled in parallel with nvcc and linked
into one shared library.
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
OUT = os.path.join(PKG, "librcx.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    *ARCH,
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-I", os.path.join(ROOT, "include"),
]


def units():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if not f.endswith(".cu")] + \
        [os.path.join(ROOT, "include", "rcx.h")]


def _obj(src):
    return os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    return _newest(units() + headers() + [os.path.abspath(__file__)]) <= os.path.getmtime(OUT)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ, exist_ok=True)
    hdr_time = _newest(headers() + [os.path.abspath(__file__)])
    procs = []
    for src in units():
        obj = _obj(src)
        if not force and os.path.exists(obj) and max(hdr_time, os.path.getmtime(src)) <= os.path.getmtime(obj):
            continue
        cmd = [nvcc, *NVCC_FLAGS, "-c", "-o", obj + ".tmp", src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, obj, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, obj, p in procs:
        out, _ = p.communicate()
        if p.returncode != 0:
            failed.append(f"{os.path.basename(src)}:\n{out}")
            continue
        if verbose:
            sys.stdout.write(out)
        os.replace(obj + ".tmp", obj)
    if failed:
        raise RuntimeError("nvcc failed:\n" + "\n".join(failed))
    cmd = [nvcc, *ARCH, "-shared", "-o", OUT + ".tmp", *[_obj(s) for s in units()]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + r.stdout + r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
